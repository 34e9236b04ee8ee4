// Adaptive block mask ("NABLA: Neighborhood Adaptive Block-Level Attention",
// section 手法: NABLA, "適応型マスク構築 (ブロックレベル・プーリング & CDF 閾値処理)"
// and "STA とのハイブリッド統合").
//
//   pool_kernel        block means of Q and K (64 tokens -> one fp32 row),
//                      float32 running sum in ascending token order, * 1/64.
//                      Q-bar row-major [BH, nb, D]; K-bar transposed
//                      [BH, D, nb] so the score kernel streams it coalesced.
//   score_cut_kernel   per (bh, 16 query blocks): pooled scores as a float32
//                      fma chain over d ascending (register-tiled FFMA; the
//                      order per output is the plain ascending chain), then
//                      per row (one warp): weights exp(s - max) in float64,
//                      integer masses floor(w * 2^40), summed exactly into a
//                      histogram over score buckets; the bucket holding the
//                      last block of the shortest descending prefix whose mass
//                      reaches p * total is ranked exactly (48-bit key: score
//                      bits, then inverted block index), and the OR with the
//                      STA window and the diagonal.  Writes the bit row and
//                      the ascending row list.
//   col_lists_kernel   transpose of the bit rows into ascending column lists.
//
// The mass sums are exact integers, so the selected set does not depend on
// the order in which threads add them.
#include "common.cuh"

namespace nabla {

// ---------------------------------------------------------------------------
// pooling
// ---------------------------------------------------------------------------
// CTA = 256 threads = (256 / CH) blocks x CH chunks of 8 features, CH = D/8.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16 *__restrict__ q,
                                                   const __nv_bfloat16 *__restrict__ k,
                                                   float *__restrict__ qbar,
                                                   float *__restrict__ kbar_t, int64_t BH,
                                                   int nb) {
    constexpr int CH = D / 8;
    constexpr int BPC = 256 / CH;  // blocks per CTA
    __shared__ float tile[BPC][D + 1];
    const int tid = threadIdx.x;
    const int c = tid % CH;
    const int bl = tid / CH;
    const int tiles_per_head = (nb + BPC - 1) / BPC;
    const int64_t cta = blockIdx.x;
    const int which = static_cast<int>(cta / (BH * tiles_per_head));  // 0: q, 1: k
    const int64_t rem = cta % (BH * tiles_per_head);
    const int64_t bh = rem / tiles_per_head;
    const int i0 = static_cast<int>(rem % tiles_per_head) * BPC;
    const int i = i0 + bl;
    const __nv_bfloat16 *x = which ? k : q;
    const int64_t N = static_cast<int64_t>(nb) * kBlk;
    const int nbp = (nb + 3) & ~3;  // row stride of the transposed K-bar

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (i < nb) {
        const int4 *src =
            reinterpret_cast<const int4 *>(x + (bh * N + static_cast<int64_t>(i) * kBlk) * D) + c;
#pragma unroll 1
        for (int r0 = 0; r0 < kBlk; r0 += 16) {
            int4 v[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = __ldg(src + (r0 + r) * CH);
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[r]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 f = __bfloat1622float2(h[e]);
                    acc[2 * e] = __fadd_rn(acc[2 * e], f.x);
                    acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], f.y);
                }
            }
        }
    }
    const float inv = 1.0f / kBlk;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = __fmul_rn(acc[e], inv);
    if (which == 0) {
        if (i < nb) {
            float4 *dst = reinterpret_cast<float4 *>(qbar + (bh * nb + i) * D + c * 8);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) tile[bl][c * 8 + e] = acc[e];
        __syncthreads();
        // write [D][nb]: each thread writes consecutive blocks of one feature
        for (int idx = tid; idx < D * BPC; idx += 256) {
            const int d = idx / BPC, b = idx % BPC;
            if (i0 + b < nb) {
                kbar_t[(bh * D + d) * nbp + i0 + b] = tile[b][d];
            } else if (i0 + b < nbp) {
                kbar_t[(bh * D + d) * nbp + i0 + b] = 0.f;  // pad column: defined, never used
            }
        }
    }
}

// ---------------------------------------------------------------------------
// fused flatten + pooling: reads Q or K in GRID order [B*h, T, H, W, D], writes
// the flattened copy [B*h, N, D] and the pooled block means in one pass.
// Block i is the P x P patch (t, py, px); its flattened token r = yy*P + xx is
// grid token (t, py*P + yy, px*P + xx).  The means are summed per feature over
// r ascending exactly as pool_kernel does over the flattened copy, so both
// paths give the same bits.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) flatten_pool_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    __nv_bfloat16 *__restrict__ qf, __nv_bfloat16 *__restrict__ kf, float *__restrict__ qbar,
    float *__restrict__ kbar_t, int64_t BH, int nb, int H, int W) {
    constexpr int CH = D / 8;
    constexpr int BPC = 256 / CH;  // blocks per CTA
    constexpr int P = 8;
    __shared__ float tile[BPC][D + 1];
    const int tid = threadIdx.x;
    const int c = tid % CH;
    const int bl = tid / CH;
    const int tiles_per_head = (nb + BPC - 1) / BPC;
    const int64_t cta = blockIdx.x;
    const int which = static_cast<int>(cta / (BH * tiles_per_head));  // 0: q, 1: k
    const int64_t rem = cta % (BH * tiles_per_head);
    const int64_t bh = rem / tiles_per_head;
    const int i0 = static_cast<int>(rem % tiles_per_head) * BPC;
    const int i = i0 + bl;
    const __nv_bfloat16 *x = which ? k : q;
    __nv_bfloat16 *xf = which ? kf : qf;
    const int64_t N = static_cast<int64_t>(nb) * kBlk;
    const int Wp = W / P, HWp = (H / P) * Wp;
    const int nbp = (nb + 3) & ~3;

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (i < nb) {
        const int t = i / HWp, py = (i % HWp) / Wp, px = i % Wp;
        // grid token of (yy, xx) = first + yy * W + xx
        const int64_t first = bh * N + (static_cast<int64_t>(t) * H + py * P) * W + px * P;
        const int4 *src = reinterpret_cast<const int4 *>(x) + c;
        int4 *dst = reinterpret_cast<int4 *>(xf + (bh * N + static_cast<int64_t>(i) * kBlk) * D) + c;
#pragma unroll 1
        for (int r0 = 0; r0 < kBlk; r0 += 16) {
            int4 v[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int rr = r0 + r;
                v[r] = __ldg(src + (first + (rr / P) * W + rr % P) * CH);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                __stcs(dst + (r0 + r) * CH, v[r]);
                const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&v[r]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 f = __bfloat1622float2(hv[e]);
                    acc[2 * e] = __fadd_rn(acc[2 * e], f.x);
                    acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], f.y);
                }
            }
        }
    }
    const float inv = 1.0f / kBlk;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = __fmul_rn(acc[e], inv);
    if (which == 0) {
        if (i < nb) {
            float4 *dst = reinterpret_cast<float4 *>(qbar + (bh * nb + i) * D + c * 8);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) tile[bl][c * 8 + e] = acc[e];
        __syncthreads();
        for (int idx = tid; idx < D * BPC; idx += 256) {
            const int d = idx / BPC, b = idx % BPC;
            if (i0 + b < nb) {
                kbar_t[(bh * D + d) * nbp + i0 + b] = tile[b][d];
            } else if (i0 + b < nbp) {
                kbar_t[(bh * D + d) * nbp + i0 + b] = 0.f;  // pad column: defined, never used
            }
        }
    }
}

// ---------------------------------------------------------------------------
// scores + CDF cut + STA + lists
// ---------------------------------------------------------------------------
constexpr int kRows = 16;       // query blocks per CTA
constexpr int kCols = 256;      // key blocks per score tile
constexpr int kDc = 8;          // features per staged K-bar slice
constexpr int kStages = 3;      // cp.async ring depth of the K-bar slices
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBuckets = 256;   // mass histogram buckets of one row
constexpr float kBucketScale = 9.0f;  // buckets per unit of (s_max - s): 256 cover 28.4
constexpr int kWarpScratch = 2048;    // bytes per warp: histogram, then the bucket's entries
constexpr int kListCap = kWarpScratch / 8;
constexpr int kMaxWords = 64;   // bit-row words of the largest row (2048 blocks)
static_assert(kStages * kDc * kCols * 4 >= kWarps * kWarpScratch, "scratch fits the ring");

struct CutParams {
    int nb, T, Hp, Wp, wt, wh, ww;
    unsigned flags;
    float p, scale;
};

__device__ __forceinline__ uint32_t order_key(float s) {
    uint32_t b = __float_as_uint(s);
    if (b == 0x80000000u) b = 0u;  // -0 ranks with +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Rank key of block j in a row: larger first = score descending, then index
// ascending.
__device__ __forceinline__ uint64_t rank_key(float s, int j) {
    return (static_cast<uint64_t>(order_key(s)) << 16) | static_cast<uint64_t>(0xFFFF - j);
}

// Integer mass floor(exp(s - smax) * 2^40), held in a double (exact: an
// integer <= 2^40; sums of up to 2^12 of them stay below 2^53, so every sum
// below is exact whatever the order of the additions).
__device__ __forceinline__ double mass_of(float s, float smax) {
    const double w = exp(static_cast<double>(s) - static_cast<double>(smax));
    return trunc(w * 1099511627776.0);  // * 2^40 is an exact scaling
}

// Histogram bucket of a score: non-decreasing as the score decreases (float
// subtraction, multiplication and truncation are all monotone), equal for
// equal scores, so the buckets cut the rank order into consecutive runs.
__device__ __forceinline__ int bucket_of(float s, float smax) {
    const float x = __fmul_rn(__fsub_rn(smax, s), kBucketScale);
    return x < static_cast<float>(kBuckets) ? __float2int_rz(x) : kBuckets - 1;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA per (bh, 16 query blocks).
//   Phase 1: the 16 x nb pooled scores into shared memory (register-tiled
//            FFMA, 4 x 4 outputs per thread; K-bar^T slices of 8 features x
//            256 blocks stream through a 3-deep cp.async ring; every output
//            is the plain fma chain over d = 0 .. D-1).
//   Phase 2: one warp per row.  The exact integer masses are summed into a
//            256-bucket histogram over (s_max - s); a scan of it finds the
//            bucket that holds the last kept block and the mass before it.
//            Only that bucket's blocks are ranked exactly (bisection over the
//            48-bit rank key, with the bucket's masses kept in shared memory),
//            so no per-block state has to live in registers.
//   Then the bit row (adaptive set OR STA window OR diagonal) and its
//   ascending list are written.
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    score_cut_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar_t,
                     CutParams prm, uint32_t *__restrict__ bits, uint16_t *__restrict__ row_idx,
                     int32_t *__restrict__ row_cnt, float *__restrict__ scores_out) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int nb = prm.nb;
    const int nbp = (nb + 3) & ~3;
    float *sS = reinterpret_cast<float *>(smem);                       // [kRows][nbp]
    float *sQt = sS + kRows * nbp;                                     // [D][kRows]
    float *sKt = sQt + D * kRows;                                      // [kStages][kDc][kCols]
    unsigned char *scratch = reinterpret_cast<unsigned char *>(sKt);   // phase 2, per warp
    uint32_t *sW = reinterpret_cast<uint32_t *>(sKt + kStages * kDc * kCols);  // [kWarps][64]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tiles = (nb + kRows - 1) / kRows;
    const int64_t bh = blockIdx.x / tiles;
    const int i0 = (blockIdx.x % tiles) * kRows;
    const int rows_here = min(kRows, nb - i0);

    // ---- phase 1
    for (int idx = tid; idx < kRows * D; idx += kThreads) {
        const int r = idx / D, d = idx % D;
        sQt[d * kRows + r] = (r < rows_here) ? qbar[(bh * nb + i0 + r) * D + d] : 0.f;
    }
    const int cg = tid % 64;  // 4 consecutive columns
    const int rg = tid / 64;  // 4 consecutive rows
    const float *kt = kbar_t + bh * static_cast<int64_t>(D) * nbp;
    constexpr int DCH = D / kDc;  // feature slices per column tile
    const int nstage = ((nb + kCols - 1) / kCols) * DCH;
    auto issue = [&](int st) {
        if (st < nstage) {
            const int j0 = (st / DCH) * kCols, d0 = (st % DCH) * kDc;
            float *dst = sKt + (st % kStages) * (kDc * kCols);
            for (int c = tid; c < kDc * kCols / 4; c += kThreads) {
                const int d = c / (kCols / 4), j = (c % (kCols / 4)) * 4;
                float *sd = dst + d * kCols + j;
                if (j0 + j < nbp) {
                    cp_async16(smem_addr(sd), kt + static_cast<int64_t>(d0 + d) * nbp + j0 + j);
                } else {
                    *reinterpret_cast<float4 *>(sd) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
        cp_async_commit();  // an empty group past the end keeps the counting uniform
    };
    float acc[4][4];
    issue(0);
    issue(1);
    for (int st = 0; st < nstage; ++st) {
        cp_async_wait<1>();  // slice st has landed (only st + 1 may be in flight)
        __syncthreads();     // ... for every thread; slot (st + 2) % 3 is free again
        issue(st + 2);
        const int j0 = (st / DCH) * kCols, d0 = (st % DCH) * kDc;
        if (d0 == 0) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
        }
        const float *sk = sKt + (st % kStages) * (kDc * kCols);
#pragma unroll
        for (int d = 0; d < kDc; ++d) {
            const float4 qv = *reinterpret_cast<const float4 *>(sQt + (d0 + d) * kRows + rg * 4);
            const float4 kv = *reinterpret_cast<const float4 *>(sk + d * kCols + cg * 4);
            const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
            const float ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(qa[a], ka[b], acc[a][b]);
        }
        if (d0 + kDc == D) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int j = j0 + cg * 4 + b;
                    if (j < nb) sS[(rg * 4 + a) * nbp + j] = __fmul_rn(acc[a][b], prm.scale);
                }
        }
    }
    cp_async_wait<0>();
    __syncthreads();  // scores complete; the ring becomes the warps' scratch

    if (scores_out != nullptr) {  // NABLA_DEBUG_SCORES: the rows as computed
        for (int idx = tid; idx < rows_here * nb; idx += kThreads) {
            const int r = idx / nb, j = idx % nb;
            scores_out[(bh * nb + i0 + r) * static_cast<int64_t>(nb) + j] = sS[r * nbp + j];
        }
    }

    // ---- phase 2: one warp per row
    const int words = (nb + 31) >> 5;
    const unsigned lt = (1u << lane) - 1u;
    uint32_t *hist = reinterpret_cast<uint32_t *>(scratch + warp * kWarpScratch);  // hi | lo
    unsigned long long *ent = reinterpret_cast<unsigned long long *>(scratch + warp * kWarpScratch);
    uint32_t *sw = sW + warp * kMaxWords;
    const int HWp = prm.Hp * prm.Wp;
    for (int r = warp; r < rows_here; r += kWarps) {
        const int i = i0 + r;
        const float *srow = sS + r * nbp;

        // row maximum
        float smax = -INFINITY;
        for (int j = lane; j < nb; j += 32) smax = fmaxf(smax, srow[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));

        // mass histogram: bucket b gets hi = sum (u >> 20) and lo = sum (u & (2^20 - 1));
        // each sum stays below 2^31 for up to 2048 blocks, so the u32 adds are exact
        for (int k = lane; k < 2 * kBuckets; k += 32) hist[k] = 0u;
        __syncwarp();
        double U = 0.0;
        for (int j = lane; j < nb; j += 32) {
            const float s = srow[j];
            const double u = mass_of(s, smax);
            if (u > 0.0) {
                const unsigned long long ui = static_cast<unsigned long long>(u);
                const int b = bucket_of(s, smax);
                atomicAdd(hist + b, static_cast<uint32_t>(ui >> 20));
                atomicAdd(hist + kBuckets + b, static_cast<uint32_t>(ui & 0xFFFFFull));
            }
            U += u;
        }
        U = warp_sum(U);
        __syncwarp();
        const double thr = static_cast<double>(prm.p) * U;

        // bucket B* holding the last kept block, and the mass before it
        double hm[kBuckets / 32], tot = 0.0;
#pragma unroll
        for (int k = 0; k < kBuckets / 32; ++k) {
            const int b = lane * (kBuckets / 32) + k;
            hm[k] = static_cast<double>(hist[b]) * 1048576.0 + static_cast<double>(hist[kBuckets + b]);
            tot += hm[k];
        }
        double incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const unsigned crossing = __ballot_sync(0xffffffffu, incl >= thr);
        int bstar = kBuckets;  // no crossing only for a non-finite row: keep it whole
        double before = 0.0;
        if (crossing != 0u) {
            const int owner = __ffs(crossing) - 1;
            int kk = 0;
            double c = incl - tot;
#pragma unroll
            for (int k = 0; k < kBuckets / 32; ++k) {
                if (c + hm[k] >= thr) break;
                c += hm[k];
                ++kk;
            }
            bstar = __shfl_sync(0xffffffffu, lane * (kBuckets / 32) + kk, owner);
            before = __shfl_sync(0xffffffffu, c, owner);
        }
        __syncwarp();  // histogram read by all lanes before the entries overwrite it

        // exact rank of the last kept block inside bucket B*: the largest rank
        // key c with before + mass(B* blocks ranked at or above c) >= thr
        uint64_t kstar = 0;
        if (bstar < kBuckets) {
            int m = 0;
            uint64_t kx = 0, kfirst = 0;
            bool have_first = false;
            for (int e = 0; e < words; ++e) {
                const int j = e * 32 + lane;
                bool in = false;
                double u = 0.0;
                float s = 0.f;
                if (j < nb) {
                    s = srow[j];
                    if (bucket_of(s, smax) == bstar) {
                        u = mass_of(s, smax);
                        in = u > 0.0;
                    }
                }
                const unsigned bal = __ballot_sync(0xffffffffu, in);
                if (bal == 0u) continue;
                if (in) {
                    const int pos = m + __popc(bal & lt);
                    if (pos < kListCap)
                        ent[pos] = (static_cast<unsigned long long>(u) << 11) |
                                   static_cast<unsigned long long>(j);
                }
                // common high bits of the bucket's rank keys narrow the search
                const int src = __ffs(bal) - 1;
                const uint64_t k0 = __shfl_sync(0xffffffffu, in ? rank_key(s, j) : 0ull, src);
                if (!have_first) {
                    kfirst = k0;
                    have_first = true;
                }
                if (in) kx |= rank_key(s, j) ^ kfirst;
                m += __popc(bal);
            }
            __syncwarp();
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kx |= __shfl_xor_sync(0xffffffffu, kx, o);
            const int top = kx ? 63 - __clzll(static_cast<long long>(kx)) : -1;
            // mass of bucket B*'s blocks with rank key >= c (exact sum)
            auto mass_ge = [&](uint64_t c) -> double {
                double a = 0.0;
                if (m <= kListCap) {
                    for (int k = lane; k < m; k += 32) {
                        const unsigned long long v = ent[k];
                        const int j = static_cast<int>(v & 0x7FFull);
                        if (rank_key(srow[j], j) >= c) a += static_cast<double>(v >> 11);
                    }
                } else {  // a bucket too full for the scratch: recompute its masses
                    for (int j = lane; j < nb; j += 32) {
                        const float s = srow[j];
                        if (bucket_of(s, smax) == bstar && rank_key(s, j) >= c)
                            a += mass_of(s, smax);
                    }
                }
                return warp_sum(a);
            };
            // invariant: before + mass_ge(kstar) >= thr (the whole bucket reaches it)
            kstar = top >= 0 ? (kfirst & ~((2ull << top) - 1ull)) : kfirst;
            for (int b = top; b >= 0; --b) {
                const uint64_t cand = kstar | (1ull << b);
                if (before + mass_ge(cand) >= thr) kstar = cand;
            }
        }

        // bit row: adaptive set, then the STA window and the diagonal
        for (int e = 0; e < words; ++e) {
            const int j = e * 32 + lane;
            bool keep = false;
            if (j < nb) {
                const float s = srow[j];
                const int b = bucket_of(s, smax);
                keep = b < bstar || (b == bstar && rank_key(s, j) >= kstar);
            }
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) sw[e] = bal;
        }
        __syncwarp();
        if (lane == 0) atomicOr(sw + (i >> 5), 1u << (i & 31));
        if (!(prm.flags & 1u)) {
            // the window clipped to the grid, enumerated block by block
            const int ti = i / HWp, hi = (i / prm.Wp) % prm.Hp, wi = i % prm.Wp;
            const int t0 = max(0, ti - prm.wt / 2), t1 = min(prm.T - 1, ti + prm.wt / 2);
            const int h0 = max(0, hi - prm.wh / 2), h1 = min(prm.Hp - 1, hi + prm.wh / 2);
            const int w0 = max(0, wi - prm.ww / 2), w1 = min(prm.Wp - 1, wi + prm.ww / 2);
            const int nh = h1 - h0 + 1, nw = w1 - w0 + 1;
            const int cells = (t1 - t0 + 1) * nh * nw;
            for (int c = lane; c < cells; c += 32) {
                const int t = t0 + c / (nh * nw), h = h0 + (c / nw) % nh, w = w0 + c % nw;
                const int j = (t * prm.Hp + h) * prm.Wp + w;
                atomicOr(sw + (j >> 5), 1u << (j & 31));
            }
        }
        __syncwarp();
        uint32_t *brow = bits + (bh * nb + i) * words;
        for (int w = lane; w < words; w += 32) brow[w] = sw[w];
        uint16_t *lst = row_idx + (bh * nb + i) * static_cast<int64_t>(nb);
        int cnt = 0;
        for (int w = 0; w < words; ++w) {
            const uint32_t word = sw[w];
            if ((word >> lane) & 1u) lst[cnt + __popc(word & lt)] = static_cast<uint16_t>(w * 32 + lane);
            cnt += __popc(word);
        }
        if (lane == 0) row_cnt[bh * nb + i] = cnt;
        __syncwarp();  // sw and the scratch are reused by the next row
    }
}

// (frame, patch row, patch column) of block j, advanced by a fixed stride
// without integer division (the emit loop visits j = lane, lane + 32, ...).
struct BlockCoord {
    int t, h, w;
    __device__ __forceinline__ BlockCoord(int j, int Hp, int Wp)
        : t(j / (Hp * Wp)), h((j / Wp) % Hp), w(j % Wp) {}
    __device__ __forceinline__ void advance(int by, int Hp, int Wp) {
        w += by;
        while (w >= Wp) {
            w -= Wp;
            if (++h == Hp) {
                h = 0;
                ++t;
            }
        }
    }
};

// STA window (section 手法: NABLA, "STA とのハイブリッド統合") in block coordinates:
// |dt| <= wt/2, |dh| <= wh/2, |dw| <= ww/2.
__device__ __forceinline__ bool in_window(const BlockCoord &a, const BlockCoord &b,
                                          const CutParams &prm) {
    return abs(a.t - b.t) <= prm.wt / 2 && abs(a.h - b.h) <= prm.wh / 2 &&
           abs(a.w - b.w) <= prm.ww / 2;
}

// ---------------------------------------------------------------------------
// masks that do not depend on the scores: p >= 1 or FULL_STA keeps every
// block; p <= 0 keeps the STA window and the diagonal (the diagonal alone with
// NO_STA).  Neither pooling nor scores are needed: one warp per row emits the
// bit row and the list directly.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) sta_emit_kernel(CutParams prm, int64_t rows,
                                                      uint32_t *__restrict__ bits,
                                                      uint16_t *__restrict__ row_idx,
                                                      int32_t *__restrict__ row_cnt) {
    const int lane = threadIdx.x & 31;
    const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;  // whole warps: rows is per warp
    const int nb = prm.nb;
    const int words = (nb + 31) >> 5;
    const int i = static_cast<int>(r % nb);
    const bool all = prm.p >= 1.0f || (prm.flags & 2u);
    const BlockCoord ci(i, prm.Hp, prm.Wp);
    BlockCoord cj(lane, prm.Hp, prm.Wp);
    uint16_t *lst = row_idx + r * static_cast<int64_t>(nb);
    int cnt = 0;
    for (int w = 0; w < words; ++w, cj.advance(32, prm.Hp, prm.Wp)) {
        const int j = w * 32 + lane;
        bool m = false;
        if (j < nb) m = all || j == i || (!(prm.flags & 1u) && in_window(ci, cj, prm));
        const unsigned ball = __ballot_sync(0xffffffffu, m);
        if (lane == 0) bits[r * words + w] = ball;
        if (m) lst[cnt + __popc(ball & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
        cnt += __popc(ball);
    }
    if (lane == 0) row_cnt[r] = cnt;
}

// ---------------------------------------------------------------------------
// column lists: transpose of the bit rows.  One CTA per (bh, 32-column word w);
// warp k takes a contiguous run of 32-row chunks.  Each chunk's 32 words are
// transposed with 32 ballots (lane c ends up holding column 32w + c of those
// rows); per-column counts of the runs are scanned across the warps in shared
// memory, then each warp writes its run's entries column by column, the lanes
// storing consecutive entries together.
// ---------------------------------------------------------------------------
constexpr int kColWarps = 8;
constexpr int kMaxChunksPerWarp = (kMaxWords + kColWarps - 1) / kColWarps;

__global__ void __launch_bounds__(kColWarps * 32) col_lists_kernel(
    const uint32_t *__restrict__ bits, uint16_t *__restrict__ col_idx,
    int32_t *__restrict__ col_cnt, int nb) {
    __shared__ int scnt[kColWarps][32];
    const int words = (nb + 31) >> 5;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t bh = blockIdx.x / words;
    const int w = static_cast<int>(blockIdx.x % words);
    const int per = (words + kColWarps - 1) / kColWarps;  // chunks per warp
    const int c0 = warp * per, c1 = min(words, c0 + per);
    uint32_t mine[kMaxChunksPerWarp];
    int cnt = 0;
#pragma unroll
    for (int cc = 0; cc < kMaxChunksPerWarp; ++cc) {
        mine[cc] = 0u;
        const int c = c0 + cc;
        if (c < c1) {
            const int i = c * 32 + lane;
            const uint32_t word = (i < nb) ? bits[(bh * nb + i) * words + w] : 0u;
            uint32_t col = 0u;
#pragma unroll
            for (int b = 0; b < 32; ++b) {
                const uint32_t t = __ballot_sync(0xffffffffu, (word >> b) & 1u);
                if (lane == b) col = t;
            }
            mine[cc] = col;
            cnt += __popc(col);
        }
    }
    scnt[warp][lane] = cnt;
    __syncthreads();
    int off = 0;
    for (int k = 0; k < warp; ++k) off += scnt[k][lane];
    const int j_lane = w * 32 + lane;
    if (warp == kColWarps - 1 && j_lane < nb) col_cnt[bh * nb + j_lane] = off + cnt;
    const unsigned lt = (1u << lane) - 1u;
    for (int b = 0; b < 32; ++b) {
        const int j = w * 32 + b;
        if (j >= nb) break;
        int o = __shfl_sync(0xffffffffu, off, b);
        uint16_t *dst = col_idx + (bh * nb + j) * static_cast<int64_t>(nb);
#pragma unroll
        for (int cc = 0; cc < kMaxChunksPerWarp; ++cc) {
            const uint32_t mw = __shfl_sync(0xffffffffu, mine[cc], b);
            if ((mw >> lane) & 1u) dst[o + __popc(mw & lt)] = static_cast<uint16_t>((c0 + cc) * 32 + lane);
            o += __popc(mw);
        }
    }
}

}  // namespace nabla

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
size_t nabla_score_cut_smem(int nb, int D) {
    const size_t nbp = (static_cast<size_t>(nb) + 3) & ~static_cast<size_t>(3);
    return sizeof(float) * (nabla::kRows * nbp + static_cast<size_t>(D) * nabla::kRows +
                            nabla::kStages * nabla::kDc * nabla::kCols) +
           sizeof(uint32_t) * nabla::kWarps * nabla::kMaxWords;
}

template <int D>
static cudaError_t launch_score_cut(dim3 grid, size_t smem, const float *qbar,
                                    const float *kbar_t, nabla::CutParams prm, uint32_t *bits,
                                    uint16_t *row_idx, int32_t *row_cnt, float *scores,
                                    cudaStream_t stream) {
    cudaError_t err = cudaFuncSetAttribute(nabla::score_cut_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(nabla::score_cut_kernel<D>,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (err != cudaSuccess) return err;
    nabla::score_cut_kernel<D><<<grid, nabla::kThreads, smem, stream>>>(qbar, kbar_t, prm, bits,
                                                                       row_idx, row_cnt, scores);
    return cudaGetLastError();
}

// q_grid/k_grid non-null: q and k are in grid order; flatten them into q/k
// (then outputs) in the same pass as the pooling.  scores non-null: also
// write the pooled scores [BH, nb, nb] (only when the mask depends on them).
cudaError_t nabla_launch_build_mask(int64_t BH, int nb, int D, int T, int Hp, int Wp, float p,
                                    float scale, int wt, int wh, int ww, unsigned flags,
                                    const void *q, const void *k, float *qbar, float *kbar_t,
                                    uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                                    uint16_t *col_idx, int32_t *col_cnt, float *scores,
                                    cudaStream_t stream, const void *q_grid, const void *k_grid) {
    using namespace nabla;
    CutParams prm{nb, T, Hp, Wp, wt, wh, ww, flags, p, scale};
    cudaError_t err;
    const bool from_grid = q_grid != nullptr;
    const int bpc = 256 / (D / 8);
    const int64_t tiles = (nb + bpc - 1) / bpc;
    const dim3 pool_grid(static_cast<unsigned>(2 * BH * tiles));
    const int words = (nb + 31) / 32;
    const dim3 col_grid(static_cast<unsigned>(BH * words));
    if (from_grid) {
        // flatten (and pool) first: the flattened copies are outputs either way
        const auto qg = static_cast<const __nv_bfloat16 *>(q_grid);
        const auto kg = static_cast<const __nv_bfloat16 *>(k_grid);
        auto qf = static_cast<__nv_bfloat16 *>(const_cast<void *>(q));
        auto kf = static_cast<__nv_bfloat16 *>(const_cast<void *>(k));
        if (D == 128)
            flatten_pool_kernel<128><<<pool_grid, 256, 0, stream>>>(qg, kg, qf, kf, qbar, kbar_t,
                                                                   BH, nb, Hp * 8, Wp * 8);
        else
            flatten_pool_kernel<64><<<pool_grid, 256, 0, stream>>>(qg, kg, qf, kf, qbar, kbar_t,
                                                                  BH, nb, Hp * 8, Wp * 8);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    if (p <= 0.0f || p >= 1.0f || (flags & 2u)) {
        // the mask does not depend on the scores
        const int64_t rows = BH * nb;
        sta_emit_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, stream>>>(
            prm, rows, bits, row_idx, row_cnt);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
        if (col_idx) {
            col_lists_kernel<<<col_grid, kColWarps * 32, 0, stream>>>(bits, col_idx, col_cnt, nb);
            err = cudaGetLastError();
        }
        return err;
    }
    if (!from_grid) {
        if (D == 128)
            pool_kernel<128><<<pool_grid, 256, 0, stream>>>(
                static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), qbar,
                kbar_t, BH, nb);
        else
            pool_kernel<64><<<pool_grid, 256, 0, stream>>>(
                static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), qbar,
                kbar_t, BH, nb);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }

    const size_t smem = nabla_score_cut_smem(nb, D);
    const dim3 grid(static_cast<unsigned>(BH * ((nb + kRows - 1) / kRows)));
    err = D == 128 ? launch_score_cut<128>(grid, smem, qbar, kbar_t, prm, bits, row_idx, row_cnt,
                                           scores, stream)
                   : launch_score_cut<64>(grid, smem, qbar, kbar_t, prm, bits, row_idx, row_cnt,
                                          scores, stream);
    if (err != cudaSuccess) return err;
    if (col_idx) {
        col_lists_kernel<<<col_grid, kColWarps * 32, 0, stream>>>(bits, col_idx, col_cnt, nb);
        err = cudaGetLastError();
    }
    return err;
}
