// Block-sparse attention forward on 5th-generation tensor cores (tcgen05,
// TMEM, TMA), head dim D = 128 or 64 (one template).
//
// "NABLA: Neighborhood Adaptive Block-Level Attention", section 手法: NABLA,
// bullet "拡張": attention is computed exactly on the kept 64 x 64 blocks.
//
// Work unit (one CTA): two query blocks of one head that are temporal
// neighbours -- the same 8 x 8 patch in frames 2u and 2u+1 -- processed
// together over the UNION of their block-mask rows, so that every K/V tile
// fetched from L2 serves 128 queries.  Each union entry carries a 2-bit
// membership; keys outside a query block's own row get probability 0 for its
// queries, so each block's result is exactly its own block-sparse attention.
//
// Per tile of two union key blocks (128 keys):
//   S = Q_pair . K_tile^T   (M = 128 queries, N = 128 keys; Q is the TMEM
//                            A operand, K the shared-memory B operand;
//                            S double-buffered in TMEM)
//   P = exp2(S * scale*log2e - m)   two softmax warpgroups: thread (g, r)
//                            owns query row r and the 64 keys of union block
//                            2t+g; the row maximum is combined through shared
//                            memory; bf16 P is written back over S in TMEM
//   O += P . V_tile          (P the TMEM A operand, V from shared memory)
// Each row keeps a reference maximum m; when a tile's maximum exceeds it by
// more than 2^8 the row moves to the new maximum and both halves rescale
// their half of the O row in TMEM and their partial sums (the exponent never
// exceeds 2^8 otherwise).
//
// Warp roles (320 threads): warp 0 builds the union list (OR of the two
// bit rows) and issues TMA loads of K and V through a 6-slot ring in MMA
// consumption order (K0 K1 V0 K2 V1 ...); warp 1 owns TMEM and one of its
// threads issues the MMAs (S(t+1) before O += P(t) V(t), so the next scores
// are computed while this tile's softmax runs); warps 2-9 are the softmax
// warpgroups (warp w serves TMEM lane quarter w % 4 and key half (w - 2) / 4).
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256 + D), Q [384, 384 + D/2).
// Key half g of a tile has its scores in columns [64 g, 64 g + 64) of the S
// buffer and its bf16 P in the first 32 of them.  A ring slot holds the two
// key blocks of a tile for each 64-feature half of D: [half h][block][64 x 64]
// bf16 at 16 KB per half (one 128-byte swizzle atom wide).
// Every wait is bounded: on expiry the CTA records a timeout in the status
// word, unwinds without further work, drains its in-flight copies and MMAs
// and frees TMEM; later CTAs of the launch see the status and do nothing.
#include "sm100.cuh"

namespace nabla {
namespace fwd100 {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kMaxNbFwd = 2048;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleAt = 8.f;  // log2 headroom before a row is rescaled
constexpr uint32_t kColO = 256, kColQ = 384;

// shared memory map (offsets from a 1024-byte aligned base) for head dim D
template <int D>
struct Layout {
    static constexpr int kHalves = D / 64;                           // 64-feature halves
    static constexpr int kRing = D == 128 ? 6 : 10;                  // K/V tiles in flight
    static constexpr uint32_t kTileBytes = 128u * D * 2;             // 128 rows x D bf16
    static constexpr uint32_t OFF_RING = 0;
    static constexpr uint32_t OFF_U = OFF_RING + kRing * kTileBytes;  // union list u16
    static constexpr uint32_t OFF_UF = OFF_U + 2 * (kMaxNbFwd + 8);   // membership per entry
    static constexpr uint32_t OFF_TM = OFF_UF + kMaxNbFwd + 8;        // membership per tile
    // [3][2][128] f32: partial row maxima by tile parity, then the partial sums
    static constexpr uint32_t OFF_RED = ((OFF_TM + kMaxNbFwd / 2 + 8 + 15) / 16) * 16;
    static constexpr uint32_t OFF_BAR = OFF_RED + 3 * 2 * 128 * 4;
    static constexpr int kNumBars = 2 * kRing + 2 + 1 + 2 + 1 + 1 + 1;
    static constexpr uint32_t OFF_INT = OFF_BAR + 8 * kNumBars;       // ints
    static constexpr uint32_t kSmemBytes = OFF_INT + 16 + 1024;       // + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
               const __nv_bfloat16 *__restrict__ q, const uint32_t *__restrict__ bits,
               __nv_bfloat16 *__restrict__ out, float *__restrict__ lse, int *__restrict__ status,
               int nb, int Hp, int Wp, int T, float c, uint32_t wait_limit, int force_timeout) {
    using L = Layout<D>;
    constexpr int kRing = L::kRing, kHalves = L::kHalves;
    constexpr uint32_t kTileBytes = L::kTileBytes;
    constexpr uint32_t OFF_U = L::OFF_U, OFF_UF = L::OFF_UF, OFF_TM = L::OFF_TM,
                       OFF_RED = L::OFF_RED, OFF_BAR = L::OFF_BAR, OFF_INT = L::OFF_INT;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
    unsigned char *sm = smem_raw + pad;
    const uint32_t sRing = raw + pad + L::OFF_RING;
    uint16_t *uList = reinterpret_cast<uint16_t *>(sm + OFF_U);
    uint8_t *uFlag = sm + OFF_UF;
    uint8_t *tileMem = sm + OFF_TM;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *kv_full = bar, *kv_empty = bar + kRing, *s_full = bar + 2 * kRing;
    // p_full[t & 1]: the eight softmax warps wrote P(t).  Two barriers, so that a
    // warp already on tile t+1 cannot complete tile t's phase for the others.
    uint64_t *q_ready = s_full + 2, *p_full = q_ready + 1, *p_empty = p_full + 2;
    uint64_t *o_done = p_empty + 1, *never = o_done + 1;
    float *red = reinterpret_cast<float *>(sm + OFF_RED);  // [slot][half][row]
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
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&kv_full[r], 1);
            mbar_init(&kv_empty[r], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(q_ready, 8);
        mbar_init(&p_full[0], 8);
        mbar_init(&p_full[1], 8);
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
        prefetch_tmap(&tk);
        prefetch_tmap(&tv);
        uint32_t seq = 0;
        auto load = [&](const CUtensorMap *tm, int t) -> bool {
            const int slot = static_cast<int>(seq % kRing);
            if (!wait_bar(&kv_empty[slot], ((seq / kRing) & 1u) ^ 1u, abort_flag, status, wait_limit))
                return false;
            mbar_expect_tx(&kv_full[slot], kTileBytes);
            const int y0 = row_base + uList[2 * t] * kBlk, y1 = row_base + uList[2 * t + 1] * kBlk;
            const uint32_t dst = sRing + slot * kTileBytes;
#pragma unroll
            for (int h = 0; h < kHalves; ++h) {
                tma_load_2d(dst + h * 16384, tm, &kv_full[slot], 64 * h, y0);
                tma_load_2d(dst + h * 16384 + 8192, tm, &kv_full[slot], 64 * h, y1);
            }
            ++seq;
            return true;
        };
        if (ntiles > 0) {
            bool ok = load(&tk, 0);
            for (int t = 1; ok && t < ntiles; ++t) ok = load(&tk, t) && load(&tv, t - 1);
            if (ok) load(&tv, ntiles - 1);
        }
        // drain: never leave with a copy in flight
        for (uint32_t s = seq > kRing ? seq - kRing : 0; s < seq; ++s)
            wait_plain(&kv_full[s % kRing], (s / kRing) & 1u, wait_limit);
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread) ----------------
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16(128, 128, 0, 0);   // Q . K^T
            constexpr uint32_t kIdPV = idesc_bf16(128, D, 0, 1);    // P . V (V MN-major)
            uint32_t seq = 0;
            auto S = [&](int t) -> bool {
                const int slot = static_cast<int>(seq % kRing);
                if (!wait_bar(&kv_full[slot], (seq / kRing) & 1u, abort_flag, status, wait_limit))
                    return false;
                tc_fence_after();
                const uint32_t b0 = sRing + slot * kTileBytes;
                const uint32_t d = tmem + (t & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ts_1(d, tmem + kColQ + 8 * kk,
                             desc_sw128(b0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), kIdS,
                             kk > 0);
                mma_commit_1(&kv_empty[slot]);
                mma_commit_1(&s_full[t & 1]);
                ++seq;
                return true;
            };
            auto PV = [&](int t) -> bool {
                const int slot = static_cast<int>(seq % kRing);
                if (!wait_bar(&kv_full[slot], (seq / kRing) & 1u, abort_flag, status, wait_limit))
                    return false;
                if (!wait_bar(&p_full[t & 1], (t >> 1) & 1, abort_flag, status, wait_limit))
                    return false;
                tc_fence_after();
                const uint32_t b0 = sRing + slot * kTileBytes;
                const uint32_t pcol = tmem + (t & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < 128 / 16; ++kk)  // keys 16kk.. at column 64(kk/4) + 8(kk%4)
                    mma_ts_1(tmem + kColO, pcol + 64 * (kk >> 2) + 8 * (kk & 3),
                             desc_sw128(b0 + kk * 2048, 16384, 1024), kIdPV, (t > 0 || kk > 0));
                mma_commit_1(&kv_empty[slot]);
                mma_commit_1(p_empty);
                ++seq;
                return true;
            };
            if (ntiles > 0 && wait_bar(q_ready, 0, abort_flag, status, wait_limit)) {
                bool ok = S(0);
                for (int t = 0; ok && t < ntiles; ++t) {
                    if (t + 1 < ntiles) ok = S(t + 1);
                    ok = ok && PV(t);
                }
            }
            mma_commit_1(o_done);  // completes once every MMA issued above has finished
            wait_plain(o_done, 0, wait_limit);
        }
    } else if (warp >= 2) {
        // ---------------- softmax: thread (g, r) = key half g, query row r ----------------
        const int wq = warp & 3;                    // TMEM lane quarter of this warp
        const int g = (warp - 2) >> 2;              // key half of the tile
        const int r = wq * 32 + lane;               // query row of the pair, 0..127
        const int h = r >> 6;                       // 0 -> block iA, 1 -> block iB
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const int ib = h ? (iB >= 0 ? iB : iA) : iA;
        const int64_t grow = bh * N + static_cast<int64_t>(ib) * kBlk + (r & 63);
        bool ok = true;
        if (force_timeout) ok = wait_bar(never, 0, abort_flag, status, 16);  // nothing arrives
        {
            // features [D/2 g, D/2 g + D/2) of the Q row -> TMEM columns
            // [D/4 g, D/4 g + D/4) of Q (the A operand of S = Q K^T)
            const uint4 *src = reinterpret_cast<const uint4 *>(q + grow * D + (D / 2) * g);
            uint32_t qv[D / 4];
#pragma unroll
            for (int e = 0; e < D / 16; ++e) {
                const uint4 v = __ldg(src + e);
                qv[4 * e] = v.x;
                qv[4 * e + 1] = v.y;
                qv[4 * e + 2] = v.z;
                qv[4 * e + 3] = v.w;
            }
            if constexpr (D == 128)
                tmem_st32(tmem + lane_base + kColQ + 32 * g, reinterpret_cast<float *>(qv));
            else
                tmem_st16(tmem + lane_base + kColQ + 16 * g, qv);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_ready);

        float m = -INFINITY, l = 0.f;  // l: partial sum over this half's keys
        for (int t = 0; t < ntiles; ++t) {
            ok = wait_bar(&s_full[t & 1], (t >> 1) & 1, abort_flag, status, wait_limit) && ok;
            tc_fence_after();
            const bool valid = (tileMem[t] >> (2 * g + h)) & 1u;  // uniform per warp
            const uint32_t scol = tmem + lane_base + (t & 1) * 128 + 64 * g;
            float s[64];
            float pmax = -INFINITY;
            if (valid) {
                tmem_ld32(scol, s);
                tmem_ld32(scol + 32, s + 32);
                tmem_wait_ld();
                // 8 chains of three-input max: 28 instructions for 56 values
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = s[e];
#pragma unroll
                for (int k = 8; k < 64; k += 2) mx8[(k >> 1) & 7] = fmax3(mx8[(k >> 1) & 7], s[k], s[k + 1]);
                pmax = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7]));
            }
            // row maximum over both halves
            red[((t & 1) * 2 + g) * 128 + r] = pmax;
            bar_sync(1, 256);
            const float tmax = c * fmaxf(pmax, red[((t & 1) * 2 + (g ^ 1)) * 128 + r]);
            // TMEM loads/stores are warp-collective (.sync.aligned): the
            // decision to move to a new reference is taken per warp (the two
            // warps serving the same rows take the same decision from the same
            // values); every lane then moves to max(m, tmax).
            if (__any_sync(0xffffffffu, tmax > m + kRescaleAt)) {
                const float mnew = fmaxf(m, tmax);
                const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mnew);
                if (__any_sync(0xffffffffu, m != -INFINITY)) {
                    // rows with earlier keys: this half of the O row moves to mnew
                    ok = wait_bar(p_empty, (t - 1) & 1, abort_flag, status, wait_limit) && ok;
                    tc_fence_after();
#pragma unroll
                    for (int part = 0; part < D / 64; ++part) {
                        float ov[32];
                        tmem_ld32(tmem + lane_base + kColO + (D / 2) * g + 32 * part, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                        tmem_st32(tmem + lane_base + kColO + (D / 2) * g + 32 * part, ov);
                    }
                    tmem_wait_st();
                }
                l *= alpha;
                m = mnew;
            }
            uint32_t pk[32];
            if (valid) {
                // pairs of keys: the exponent s c - m of each is one packed
                // fused multiply-add; four packed partial sums
                const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m, -m);
                uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                    const uint64_t x = f2_fma(f2_pack(s[k], s[k + 1]), c2, nm2);
                    const float p0 = fast_exp2(f2_lo(x));
                    const float p1 = fast_exp2(f2_hi(x));
                    ls2[(k >> 1) & 3] = f2_add(ls2[(k >> 1) & 3], f2_pack(p0, p1));
                    pk[k >> 1] = pack_bf16(p0, p1);
                }
                const uint64_t lsum = f2_add(f2_add(ls2[0], ls2[1]), f2_add(ls2[2], ls2[3]));
                l += f2_lo(lsum) + f2_hi(lsum);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = 0u;
            }
            // bf16 P over the first 32 columns of this half's scores
            tmem_st32(scol, reinterpret_cast<float *>(pk));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t & 1]);
        }
        // ---------------- epilogue: half g writes features [D/2 g, D/2 g + D/2) ----------------
        if (ok && ntiles > 0) ok = wait_bar(o_done, 0, abort_flag, status, wait_limit);
        tc_fence_after();
        red[(4 + g) * 128 + r] = l;  // own slot: the partner may still read the last maxima
        bar_sync(1, 256);
        l += red[(4 + (g ^ 1)) * 128 + r];
        // warp-uniform: every lane of the warp takes the same branches around
        // the collective TMEM loads
        const bool aborted = __any_sync(0xffffffffu, *abort_flag != 0);
        const bool have = (h == 0 || iB >= 0) && !aborted;
        const bool read_o = have && ntiles > 0 && __all_sync(0xffffffffu, ok);
        if (have) {
            const bool live = read_o && l > 0.f;
            if (lse != nullptr && g == 0) lse[grow] = live ? (m + log2f(l)) * kLn2 : -INFINITY;
            const float inv = live ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = out + grow * D + (D / 2) * g;
#pragma unroll
            for (int part = 0; part < D / 64; ++part) {
                float ov[32];
                if (read_o) {
                    tmem_ld32(tmem + lane_base + kColO + (D / 2) * g + 32 * part, ov);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = 0.f;
                }
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    uint4 w;
                    w.x = pack_bf16(ov[8 * e8] * inv, ov[8 * e8 + 1] * inv);
                    w.y = pack_bf16(ov[8 * e8 + 2] * inv, ov[8 * e8 + 3] * inv);
                    w.z = pack_bf16(ov[8 * e8 + 4] * inv, ov[8 * e8 + 5] * inv);
                    w.w = pack_bf16(ov[8 * e8 + 6] * inv, ov[8 * e8 + 7] * inv);
                    *reinterpret_cast<uint4 *>(dst + 32 * part + 8 * e8) = w;
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

// [rows, D] bf16 row-major (D = 64 or 128), boxes of 64 rows x 64 features,
// 128-byte swizzle
bool nabla_make_tmap_rows(CUtensorMap *m, const void *base, uint64_t rows, int D) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_fwd(int64_t BH, int nb, int Hp, int Wp, int T, float scale,
                              const void *q, const void *k, const void *v, const uint32_t *bits,
                              void *o, float *lse, int *status, int force_timeout,
                              cudaStream_t stream) {
    using namespace nabla::fwd100;
    constexpr uint32_t kSmem = Layout<D>::kSmemBytes;
    const uint64_t rows = static_cast<uint64_t>(BH) * nb * nabla::kBlk;
    if (rows >= (1ull << 31) || nb > kMaxNbFwd) return cudaErrorInvalidValue;
    CUtensorMap mk, mv;
    if (!nabla_make_tmap_rows(&mk, k, rows, D) || !nabla_make_tmap_rows(&mv, v, rows, D))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(fwd_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kSmem));
    if (err != cudaSuccess) return err;
    const int64_t groups = static_cast<int64_t>((T + 1) / 2) * Hp * Wp;
    const float c = scale * 1.4426950408889634f;
    const uint32_t limit = 1000000000u;  // 1 s per wait
    fwd_kernel<D><<<static_cast<unsigned>(BH * groups), kThreads, kSmem, stream>>>(
        mk, mv, static_cast<const __nv_bfloat16 *>(q), bits, static_cast<__nv_bfloat16 *>(o), lse,
        status, nb, Hp, Wp, T, c, limit, force_timeout);
    return cudaGetLastError();
}

cudaError_t nabla_launch_attn_fwd_sm100(int64_t BH, int nb, int D, int Hp, int Wp, int T,
                                        float scale, const void *q, const void *k, const void *v,
                                        const uint32_t *bits, void *o, float *lse, int *status,
                                        int force_timeout, cudaStream_t stream) {
    if (D == 128)
        return launch_fwd<128>(BH, nb, Hp, Wp, T, scale, q, k, v, bits, o, lse, status,
                               force_timeout, stream);
    if (D == 64)
        return launch_fwd<64>(BH, nb, Hp, Wp, T, scale, q, k, v, bits, o, lse, status,
                              force_timeout, stream);
    return cudaErrorInvalidValue;
}
