// Block-sparse attention forward on 5th-generation tensor cores (tcgen05,
// TMEM, TMA), head dim 128.
//
// "NABLA: Neighborhood Adaptive Block-Level Attention", section 手法: NABLA,
// bullet "拡張": attention is computed exactly on the kept 64 x 64 blocks.
//
// Work unit (one CTA): two query blocks of one head that are temporal
// neighbours -- the same 8 x 8 patch in frames 2u and 2u+1 -- processed
// together over the UNION of their block-mask rows, so that every K/V tile
// fetched from L2 serves 128 queries.  Each union entry carries a 2-bit
// membership; keys outside a member's own row get probability 0 for that
// member, so each member's result is exactly its own block-sparse attention.
//
// Per tile of two union key blocks (128 keys), with S and O transposed so
// that the 128 keys / 128 features fill the M = 128 tensor-core datapath:
//   S^T[128 keys x 128 queries]   = K_tile . Q_pair^T          (TMEM, fp32)
//   P^T = exp2(S^T * scale*log2e - m_q)  (bf16, SMEM; softmax warpgroups,
//                                         one thread per key row)
//   O^T[128 features x 128 q]    += V_tile^T . P^T             (TMEM, fp32)
// The reference m_q of each query column is the exact column maximum of the
// first tile holding keys of that query's block; later tiles only check that
// no exponent exceeds 2^64 and, if one would, rescale O^T and the row sums
// (a column maximum, then O^T *= 2^(m_old - m_new)).  Row sums are kept per
// key row and reduced across threads once at the end.
//
// Warp roles (384 threads): warp 0 builds the union list (OR of the two
// bit rows) and issues TMA loads; warp 1 owns TMEM and issues the MMAs;
// warps 4-7 / 8-11 are the softmax warpgroups of the two member blocks.
// K and V tiles stream through a 4-slot ring of 32 KB slots in MMA
// consumption order (K0 K1 V0 K2 V1 ...).  S is double-buffered in TMEM.
// Every wait is bounded: on expiry the CTA records a timeout in the status
// word, unwinds without further work, drains its in-flight copies and MMAs
// and frees TMEM.
#include "sm100.cuh"

namespace nabla {
namespace fwd100 {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kRing = 4;
constexpr uint32_t kTileBytes = 32768;  // 128 rows x 128 bf16
constexpr int kD = 128;
constexpr int kMaxNbFwd = 2048;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleAt = 64.f;  // log2 headroom before O is rescaled

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_Q = 0;                                     // 32 KB
constexpr uint32_t OFF_RING = 32768;                              // kRing x 32 KB
constexpr uint32_t OFF_P = OFF_RING + kRing * kTileBytes;         // 32 KB
constexpr uint32_t OFF_U = OFF_P + 32768;                         // union list u16
constexpr uint32_t OFF_UF = OFF_U + 2 * (kMaxNbFwd + 8);          // membership per entry
constexpr uint32_t OFF_TM = OFF_UF + kMaxNbFwd + 8;               // membership per tile
constexpr uint32_t OFF_M = OFF_TM + kMaxNbFwd / 2 + 8;            // m [2][64]
constexpr uint32_t OFF_A = ((OFF_M + 512 + 15) / 16) * 16;        // alpha [2][64]
constexpr uint32_t OFF_RED = OFF_A + 512;                         // [2][4][64]
constexpr uint32_t OFF_L = OFF_RED + 2048;                        // [2][64]
constexpr uint32_t OFF_BAR = ((OFF_L + 512 + 7) / 8) * 8;         // barriers
constexpr int kNumBars = 1 + 2 * kRing + 2 + 2 + 1 + 1 + 1 + 1;
constexpr uint32_t OFF_INT = OFF_BAR + 8 * kNumBars;              // ints
constexpr uint32_t kSmemBytes = OFF_INT + 16 + 1024;              // + alignment slack

// Transposed warp reduction of 32 values per lane: afterwards lane l holds
// the reduction over the warp of column l (in v[0]).
template <bool MAX>
__device__ __forceinline__ float warp_columns32(float (&v)[32], int lane) {
#pragma unroll
    for (int step = 16; step >= 1; step >>= 1) {
        const bool hi = (lane & step) != 0;
#pragma unroll
        for (int i = 0; i < step; ++i) {
            const float send = hi ? v[i] : v[i + step];
            const float keep = hi ? v[i + step] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, step);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const uint32_t *__restrict__ bits,
               __nv_bfloat16 *__restrict__ out, float *__restrict__ lse, int *__restrict__ status,
               int nb, int Hp, int Wp, int T, float c, uint32_t wait_limit, int force_timeout) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
    unsigned char *sm = smem_raw + pad;
    const uint32_t sbase = raw + pad;
    const uint32_t sQ = sbase + OFF_Q, sRing = sbase + OFF_RING, sP = sbase + OFF_P;
    uint16_t *uList = reinterpret_cast<uint16_t *>(sm + OFF_U);
    uint8_t *uFlag = sm + OFF_UF;
    uint8_t *tileMem = sm + OFF_TM;
    float *sM = reinterpret_cast<float *>(sm + OFF_M);
    float *sAlpha = reinterpret_cast<float *>(sm + OFF_A);
    float *sRed = reinterpret_cast<float *>(sm + OFF_RED);
    float *sLsum = reinterpret_cast<float *>(sm + OFF_L);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *q_full = bar, *kv_full = bar + 1, *kv_empty = bar + 1 + kRing;
    uint64_t *s_full = bar + 1 + 2 * kRing, *s_empty = s_full + 2, *p_full = s_empty + 2;
    uint64_t *p_empty = p_full + 1, *o_done = p_empty + 1, *never = o_done + 1;
    int *sInt = reinterpret_cast<int *>(sm + OFF_INT);  // [0] tmem base [1] tiles [2] abort
    volatile int *abort_flag = sInt + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int words = (nb + 31) >> 5;
    const int HW = Hp * Wp;
    const int G = ((T + 1) >> 1) * HW;
    const int64_t bh = blockIdx.x / G;
    const int g = static_cast<int>(blockIdx.x % G);
    const int iA = 2 * (g / HW) * HW + g % HW;
    const int iB = (2 * (g / HW) + 1 < T) ? iA + HW : -1;
    const int64_t N = static_cast<int64_t>(nb) * kBlk;
    const int row_base = static_cast<int>(bh * N);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&kv_full[r], 1);
            mbar_init(&kv_empty[r], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 8);
        }
        mbar_init(p_full, 8);
        mbar_init(p_empty, 1);
        mbar_init(o_done, 1);
        mbar_init(never, 1);
        // a CTA of this launch already gave up: do no work at all
        sInt[2] = *reinterpret_cast<volatile int *>(status) != 0 ? 1 : 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(reinterpret_cast<uint32_t *>(&sInt[0]), 512);
        tmem_relinquish();
    }
    if (warp == 0) {
        // union of the two bit rows, ascending, with 2-bit membership
        const uint32_t *ra = bits + (bh * nb + iA) * words;
        const uint32_t *rb = iB >= 0 ? bits + (bh * nb + iB) * words : nullptr;
        const int U = union_bits(ra, rb, words, uList, uFlag, lane);
        const int ntiles = (U + 1) >> 1;
        for (int t = lane; t < ntiles; t += 32) {
            const int f0 = uFlag[2 * t];
            const int f1 = (2 * t + 1 < U) ? uFlag[2 * t + 1] : 0;
            tileMem[t] = static_cast<uint8_t>(f0 | (f1 << 2));
        }
        if (lane == 0) {
            if (U & 1) uList[U] = uList[U - 1];  // pad the last tile with a real block
            sInt[1] = ntiles;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(sInt[0]);
    const int ntiles = *abort_flag ? 0 : sInt[1];

    if (warp == 0 && lane == 0) {
        // ---------------- producer: TMA loads ----------------
        prefetch_tmap(&tq);
        prefetch_tmap(&tk);
        prefetch_tmap(&tv);
        const int ya = row_base + iA * kBlk, yb = row_base + (iB >= 0 ? iB : iA) * kBlk;
        mbar_expect_tx(q_full, 4 * 8192);
        tma_load_2d(sQ, &tq, q_full, 0, ya);
        tma_load_2d(sQ + 8192, &tq, q_full, 0, yb);
        tma_load_2d(sQ + 16384, &tq, q_full, 64, ya);
        tma_load_2d(sQ + 24576, &tq, q_full, 64, yb);
        uint32_t seq = 0;
        auto load = [&](const CUtensorMap *tm, int t) -> bool {
            const int slot = static_cast<int>(seq % kRing);
            if (!wait_bar(&kv_empty[slot], ((seq / kRing) & 1u) ^ 1u, abort_flag, status, wait_limit))
                return false;
            mbar_expect_tx(&kv_full[slot], kTileBytes);
            const int y0 = row_base + uList[2 * t] * kBlk, y1 = row_base + uList[2 * t + 1] * kBlk;
            const uint32_t dst = sRing + slot * kTileBytes;
            tma_load_2d(dst, tm, &kv_full[slot], 0, y0);
            tma_load_2d(dst + 8192, tm, &kv_full[slot], 0, y1);
            tma_load_2d(dst + 16384, tm, &kv_full[slot], 64, y0);
            tma_load_2d(dst + 24576, tm, &kv_full[slot], 64, y1);
            ++seq;
            return true;
        };
        if (ntiles > 0) {
            bool ok = load(&tk, 0);
            for (int t = 1; ok && t < ntiles; ++t) ok = load(&tk, t) && load(&tv, t - 1);
            if (ok) load(&tv, ntiles - 1);
        }
        // drain: never leave with a copy in flight
        wait_plain(q_full, 0, wait_limit);
        for (uint32_t s = seq > kRing ? seq - kRing : 0; s < seq; ++s)
            wait_plain(&kv_full[s % kRing], (s / kRing) & 1u, wait_limit);
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t kIdPV = idesc_bf16(128, 128, 1, 1);
            uint32_t seq = 0;
            auto S = [&](int t) -> bool {
                const int slot = static_cast<int>(seq % kRing);
                if (!wait_bar(&kv_full[slot], (seq / kRing) & 1u, abort_flag, status, wait_limit))
                    return false;
                if (!wait_bar(&s_empty[t & 1], ((t >> 1) & 1) ^ 1, abort_flag, status, wait_limit))
                    return false;
                tc_fence_after();
                const uint32_t a0 = sRing + slot * kTileBytes;
                const uint32_t d = tmem + (t & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(d, desc_sw128(a0 + off, 16, 1024), desc_sw128(sQ + off, 16, 1024), kIdS,
                           kk > 0);
                }
                mma_commit(&kv_empty[slot]);
                mma_commit(&s_full[t & 1]);
                ++seq;
                return true;
            };
            auto PV = [&](int u) -> bool {
                const int slot = static_cast<int>(seq % kRing);
                if (!wait_bar(&kv_full[slot], (seq / kRing) & 1u, abort_flag, status, wait_limit))
                    return false;
                if (!wait_bar(p_full, u & 1, abort_flag, status, wait_limit)) return false;
                tc_fence_after();
                const uint32_t a0 = sRing + slot * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 128 / 16; ++kk)
                    mma_ss(tmem + 256, desc_sw128(a0 + kk * 2048, 16384, 1024),
                           desc_sw128(sP + kk * 2048, 16384, 1024), kIdPV, (u > 0 || kk > 0));
                mma_commit(&kv_empty[slot]);
                mma_commit(p_empty);
                ++seq;
                return true;
            };
            if (ntiles > 0 && wait_bar(q_full, 0, abort_flag, status, wait_limit)) {
                bool ok = S(0);
                for (int t = 1; ok && t < ntiles; ++t) ok = S(t) && PV(t - 1);
                if (ok) PV(ntiles - 1);
            }
            mma_commit(o_done);  // completes once every MMA issued above has finished
            wait_plain(o_done, 0, wait_limit);
        }
    } else if (warp >= 4) {
        // ---------------- softmax warpgroups ----------------
        const int h = (warp - 4) >> 2;  // member: 0 -> block iA, 1 -> block iB
        const int wq = warp & 3;        // TMEM lane quarter
        const int tw = wq * 32 + lane;  // key row of the tile, 0..127
        const int hf = tw >> 6;         // which of the tile's two key blocks
        const int barid = 1 + h;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        float *mrow = sM + h * 64;
        float l[64];
#pragma unroll
        for (int q = 0; q < 64; ++q) l[q] = 0.f;
        bool init = false;
        bool ok = true;
        if (force_timeout) ok = wait_bar(never, 0, abort_flag, status, 16);  // nothing arrives
        // After an abort every wait returns at once; the loop still runs out with
        // the same control flow in all 128 threads, so the warpgroup's named
        // barriers always match.
        for (int t = 0; t < ntiles; ++t) {
            ok = wait_bar(&s_full[t & 1], (t >> 1) & 1, abort_flag, status, wait_limit) && ok;
            tc_fence_after();
            const uint32_t mem = tileMem[t];
            const bool valid = (mem >> (2 * hf + h)) & 1u;
            const bool anyv = ((mem >> h) & 1u) | ((mem >> (2 + h)) & 1u);
            const uint32_t saddr = tmem + lane_base + (t & 1) * 128 + h * 64;
            float p[64];
            if (!anyv) {
#pragma unroll
                for (int q = 0; q < 64; ++q) p[q] = 0.f;
            } else {
                bool need = !init;
                if (init) {
                    tmem_ld32(saddr, p);
                    tmem_ld32(saddr + 32, p + 32);
                    tmem_wait_ld();
                    float xm8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) xm8[e] = -INFINITY;
#pragma unroll
                    for (int q4 = 0; q4 < 16; ++q4) {
                        const float4 m4 = reinterpret_cast<const float4 *>(mrow)[q4];
                        const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x = fmaf(p[4 * q4 + e], c, -mm[e]);
                            xm8[(4 * q4 + e) & 7] = fmaxf(xm8[(4 * q4 + e) & 7], x);
                            p[4 * q4 + e] = valid ? fast_exp2(x) : 0.f;
                        }
                    }
                    const float xm = fmaxf(fmaxf(fmaxf(xm8[0], xm8[1]), fmaxf(xm8[2], xm8[3])),
                                           fmaxf(fmaxf(xm8[4], xm8[5]), fmaxf(xm8[6], xm8[7])));
                    need = bar_or(barid, 128, valid && xm > kRescaleAt);
                }
                if (need) {
                    // column maxima of this tile over the member's key rows
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tmem_ld32(saddr + 32 * half, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q) v[q] = valid ? v[q] : -INFINITY;
                        sRed[(h * 4 + wq) * 64 + 32 * half + lane] = warp_columns32<true>(v, lane);
                    }
                    bar_sync(barid, 128);
                    if (tw < 64) {
                        float mx = sRed[(h * 4) * 64 + tw];
#pragma unroll
                        for (int w = 1; w < 4; ++w) mx = fmaxf(mx, sRed[(h * 4 + w) * 64 + tw]);
                        const float mnew = init ? fmaxf(mrow[tw], mx * c) : mx * c;
                        sAlpha[h * 64 + tw] = init ? fast_exp2(mrow[tw] - mnew) : 0.f;
                        mrow[tw] = mnew;
                    }
                    bar_sync(barid, 128);
                    if (init) {
                        // O^T and the row sums move to the new reference
                        ok = wait_bar(p_empty, (t - 1) & 1, abort_flag, status, wait_limit) && ok;
                        tc_fence_after();
                        const uint32_t oaddr = tmem + lane_base + 256 + h * 64;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            float ov[32];
                            tmem_ld32(oaddr + 32 * half, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int q = 0; q < 32; ++q) ov[q] *= sAlpha[h * 64 + 32 * half + q];
                            tmem_st32(oaddr + 32 * half, ov);
                        }
                        tmem_wait_st();
#pragma unroll
                        for (int q = 0; q < 64; ++q) l[q] *= sAlpha[h * 64 + q];
                    }
                    init = true;
                    tmem_ld32(saddr, p);
                    tmem_ld32(saddr + 32, p + 32);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 16; ++q4) {
                        const float4 m4 = reinterpret_cast<const float4 *>(mrow)[q4];
                        const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            p[4 * q4 + e] = valid ? fast_exp2(fmaf(p[4 * q4 + e], c, -mm[e])) : 0.f;
                    }
                }
#pragma unroll
                for (int q = 0; q < 64; ++q) l[q] += p[q];
            }
            // S buffer consumed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[t & 1]);
            // P^T row -> shared memory once PV(t-1) has released the buffer
            if (t > 0) ok = wait_bar(p_empty, (t - 1) & 1, abort_flag, status, wait_limit) && ok;
            const uint32_t prow = sP + h * 16384 + tw * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint32_t a = pack_bf16(p[8 * cc + 0], p[8 * cc + 1]);
                const uint32_t b = pack_bf16(p[8 * cc + 2], p[8 * cc + 3]);
                const uint32_t d = pack_bf16(p[8 * cc + 4], p[8 * cc + 5]);
                const uint32_t e = pack_bf16(p[8 * cc + 6], p[8 * cc + 7]);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                                 prow + ((cc ^ (tw & 7)) << 4)),
                             "r"(a), "r"(b), "r"(d), "r"(e)
                             : "memory");
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ---------------- epilogue ----------------
        if (ok && ntiles > 0) ok = wait_bar(o_done, 0, abort_flag, status, wait_limit);
        tc_fence_after();
        // row sums: reduce the per-key-row partials across the warpgroup
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = l[32 * half + q];
            sRed[(h * 4 + wq) * 64 + 32 * half + lane] = warp_columns32<false>(v, lane);
        }
        bar_sync(barid, 128);
        if (tw < 64) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) s += sRed[(h * 4 + w) * 64 + tw];
            sLsum[h * 64 + tw] = s;
        }
        bar_sync(barid, 128);
        const bool have = (h == 0 || iB >= 0) && !*abort_flag;
        if (have) {
            const int ib = h ? iB : iA;
            const int64_t row0 = bh * N + static_cast<int64_t>(ib) * kBlk;
            const bool live = ok && ntiles > 0 && init;
            if (lse != nullptr && tw < 64) {
                const float L = sLsum[h * 64 + tw];
                lse[row0 + tw] = (live && L > 0.f) ? (mrow[tw] + log2f(L)) * kLn2 : -INFINITY;
            }
            const uint32_t oaddr = tmem + lane_base + 256 + h * 64;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float ov[32];
                if (live) {
                    tmem_ld32(oaddr + 32 * half, ov);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) ov[q] = 0.f;
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float L = sLsum[h * 64 + 32 * half + q];
                    const float val = L > 0.f ? ov[q] / L : 0.f;
                    out[(row0 + 32 * half + q) * kD + tw] = __float2bfloat16_rn(val);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace fwd100
}  // namespace nabla

// ---------------------------------------------------------------------------
// host launcher
// ---------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

}  // namespace

// [rows, 128] bf16 row-major, boxes of 64 rows x 64 features, 128-byte swizzle
bool nabla_make_tmap_rows128(CUtensorMap *m, const void *base, uint64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {128, rows};
    const cuuint64_t strides[1] = {128 * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t nabla_fwd_sm100_smem() { return nabla::fwd100::kSmemBytes; }

cudaError_t nabla_launch_attn_fwd_sm100(int64_t BH, int nb, int Hp, int Wp, int T, float scale,
                                        const void *q, const void *k, const void *v,
                                        const uint32_t *bits, void *o, float *lse, int *status,
                                        int force_timeout, cudaStream_t stream) {
    using namespace nabla::fwd100;
    const uint64_t rows = static_cast<uint64_t>(BH) * nb * nabla::kBlk;
    if (rows >= (1ull << 31) || nb > kMaxNbFwd) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!nabla_make_tmap_rows128(&mq, q, rows) || !nabla_make_tmap_rows128(&mk, k, rows) ||
        !nabla_make_tmap_rows128(&mv, v, rows))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kSmemBytes));
    if (err != cudaSuccess) return err;
    const int64_t groups = static_cast<int64_t>((T + 1) / 2) * Hp * Wp;
    const float c = scale * 1.4426950408889634f;
    const uint32_t limit = 1u << 20;  // polls (>= 128 ns apart after the first 32): >= 0.1 s
    fwd_kernel<<<static_cast<unsigned>(BH * groups), kThreads, kSmemBytes, stream>>>(
        mq, mk, mv, bits, static_cast<__nv_bfloat16 *>(o), lse, status, nb, Hp, Wp, T, c, limit,
        force_timeout);
    return cudaGetLastError();
}
