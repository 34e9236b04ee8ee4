// Adaptive block mask ("NABLA: Neighborhood Adaptive Block-Level Attention",
// section 手法: NABLA, "適応型マスク構築 (ブロックレベル・プーリング & CDF 閾値処理)"
// and "STA とのハイブリッド統合").
//
//   pool_kernel        block means of Q and K (64 tokens -> one fp32 row),
//                      float32 running sum in ascending token order, * 1/64.
//                      Q-bar row-major [BH, nb, D]; K-bar transposed
//                      [BH, D, nb] so the score kernel streams it coalesced.
//   score_cut_kernel   per (bh, 8 query blocks): pooled scores as a float32
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
#include <algorithm>

#include "common.cuh"
#include "exp_nonpos.cuh"

namespace nabla {

// ---------------------------------------------------------------------------
// pooling
// ---------------------------------------------------------------------------
// A tile = 256 threads = (256 / CH) blocks x CH chunks of 8 features,
// CH = D/8; tile index cta = which * BH * tiles + bh * tiles + tile (which 0:
// Q, 1: K).  `tile` is [256 / CH][D + 1] floats of shared memory.
template <int D>
__device__ __forceinline__ void pool_tile(const __nv_bfloat16 *__restrict__ q,
                                          const __nv_bfloat16 *__restrict__ k,
                                          float *__restrict__ qbar, float *__restrict__ kbar_t,
                                          int64_t BH, int nb, int64_t cta,
                                          float (*tile)[D + 1]) {
    constexpr int CH = D / 8;
    constexpr int BPC = 256 / CH;  // blocks per tile
    const int tid = threadIdx.x;
    const int c = tid % CH;
    const int bl = tid / CH;
    const int tiles_per_head = (nb + BPC - 1) / BPC;
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

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16 *__restrict__ q,
                                                   const __nv_bfloat16 *__restrict__ k,
                                                   float *__restrict__ qbar,
                                                   float *__restrict__ kbar_t, int64_t BH,
                                                   int nb) {
    __shared__ float tile[256 / (D / 8)][D + 1];
    pool_tile<D>(q, k, qbar, kbar_t, BH, nb, blockIdx.x, tile);
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
__device__ __forceinline__ void flatten_pool_tile(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    __nv_bfloat16 *__restrict__ qf, __nv_bfloat16 *__restrict__ kf, float *__restrict__ qbar,
    float *__restrict__ kbar_t, int64_t BH, int nb, int H, int W, int64_t cta,
    float (*tile)[D + 1]) {
    constexpr int CH = D / 8;
    constexpr int BPC = 256 / CH;  // blocks per tile
    constexpr int P = 8;
    const int tid = threadIdx.x;
    const int c = tid % CH;
    const int bl = tid / CH;
    const int tiles_per_head = (nb + BPC - 1) / BPC;
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

template <int D>
__global__ void __launch_bounds__(256) flatten_pool_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    __nv_bfloat16 *__restrict__ qf, __nv_bfloat16 *__restrict__ kf, float *__restrict__ qbar,
    float *__restrict__ kbar_t, int64_t BH, int nb, int H, int W) {
    __shared__ float tile[256 / (D / 8)][D + 1];
    flatten_pool_tile<D>(q, k, qf, kf, qbar, kbar_t, BH, nb, H, W, blockIdx.x, tile);
}

// ---------------------------------------------------------------------------
// scores + CDF cut + STA + lists
// ---------------------------------------------------------------------------
constexpr int kRows = 8;        // query blocks per CTA (one per warp)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;          // bins of one row's mass histogram
constexpr int kHistWords = 2 * kBins;  // per warp: hi and lo u32 sums per bin
constexpr int kMaxWords = 64;       // bit-row words of the largest row (2048 blocks)
constexpr int kCand = 64;           // candidates ranked exactly by one warp at once
constexpr int kPre = 8;             // features of K-bar prefetched ahead in registers

struct CutParams {
    int nb, T, Hp, Wp, wt, wh, ww;
    unsigned flags;
    float p, scale;
    int mode;   // 0: CDF cut at p (NABLA); 1: logit threshold tau (DynamicRad)
    float tau;  // mode 1: keep s_ij with max_j s_ij - s_ij <= tau (float32)
};

// Completes one bit row held in a warp's shared words sw[0 .. words) (the
// selected blocks already set): ORs in the diagonal and the STA window
// (section 手法: NABLA, "STA とのハイブリッド統合": |dt| <= wt/2, |dh| <= wh/2,
// |dw| <= ww/2 in block coordinates, truncated at the grid border; enumerated
// block by block over the clipped window), then writes the bit row, the
// ascending row list and its count.  Called by all 32 lanes of the warp.
__device__ __forceinline__ void finish_row(const CutParams &prm, int64_t bh, int i, uint32_t *sw,
                                           uint32_t *__restrict__ bits,
                                           uint16_t *__restrict__ row_idx,
                                           int32_t *__restrict__ row_cnt) {
    const int lane = threadIdx.x & 31, nb = prm.nb, words = (nb + 31) >> 5;
    const unsigned lt = (1u << lane) - 1u;
    __syncwarp();
    if (lane == 0) atomicOr(sw + (i >> 5), 1u << (i & 31));
    if (!(prm.flags & 1u)) {
        const int HWp = prm.Hp * prm.Wp;
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
    __syncwarp();  // sw is reused by the warp's next row
}

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
// below is exact whatever the order of the additions).  s = -inf gives 0.
__device__ __forceinline__ double mass_of(float s, float smax) {
    const double w = exp_nonpos(static_cast<double>(s) - static_cast<double>(smax));
    return trunc(w * 1099511627776.0);  // * 2^40 is an exact scaling
}

// 24-bit bucket key of a score: floor(y * 2^16) with y = (s_max - s) * g in
// float32 (g > 0 fixed for the row), saturated at 2^24 - 1.  Float
// subtraction and multiplication by a positive constant are monotone and
// scaling by 2^16 is exact, so the key never decreases as the score decreases
// and equal scores share it: its bytes, most significant first, cut the rank
// order into consecutive runs at three levels of refinement.
__device__ __forceinline__ uint32_t ykey(float s, float smax, float g) {
    const float y = __fmul_rn(__fsub_rn(smax, s), g);
    return y < 256.0f ? __float2uint_rz(__fmul_rn(y, 65536.0f)) : 0xFFFFFFu;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
    const uint32_t hi = __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(v >> 32));
    const uint32_t lo = __reduce_max_sync(
        0xffffffffu, static_cast<uint32_t>(v >> 32) == hi ? static_cast<uint32_t>(v) : 0u);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Bin b holds hi = sum (u >> 20) and lo = sum (u & (2^20 - 1)); with masses
// u <= 2^40 each stays below 2^31 for up to 2048 blocks, so the u32 sums are
// exact (and cheaper than 64-bit shared atomics).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t b, double u) {
    const unsigned long long ui = static_cast<unsigned long long>(u);
    atomicAdd(hist + b, static_cast<uint32_t>(ui >> 20));
    atomicAdd(hist + kBins + b, static_cast<uint32_t>(ui & 0xFFFFFull));
}

// One CTA per (bh, 8 query blocks), three CTAs per SM.
//   Phase 1: the 8 x nb pooled scores into shared memory.  Thread t owns
//            the column pairs (2t, 2t + 1), (2t + 512, 2t + 513), ...; for each
//            it runs the 16 fma chains (8 rows x 2 columns) over d = 0 .. D-1
//            as packed fma.rn.f32x2 on row pairs (each lane rounds like fmaf),
//            the query means broadcast from shared memory and the K-bar^T
//            column pair read from L2 with 8 features prefetched in registers;
//            then times scale.
//   Phase 2: one warp per row.  Exact integer masses are summed into a
//            256-bin histogram over the top byte of the bucket key (bins
//            spread over the row's own score range); its scan gives the bin
//            holding the last kept block and the mass before it.  Blocks in
//            lower bins are kept, in higher bins dropped; the bin's own blocks
//            are refined by the key's next byte (at most three levels) until
//            at most 64 remain, which are ranked exactly by their 48-bit rank
//            keys against each other.  (Runs of equal scores that no byte can
//            split are resolved by score group, lowest index first.)
//   Then the bit row (adaptive set OR STA window OR diagonal) and its
//   ascending list are written.
// Rows [i0, i0 + 8) of head bh; `smem` is nabla_score_cut_smem() bytes.  The
// pooled means are read through L2 (ld.global.cg), so a tile may run in the
// same launch that wrote them.
template <int D>
__device__ __forceinline__ void score_cut_tile(const float *__restrict__ qbar,
                                               const float *__restrict__ kbar_t,
                                               const CutParams &prm, uint32_t *__restrict__ bits,
                                               uint16_t *__restrict__ row_idx,
                                               int32_t *__restrict__ row_cnt,
                                               float *__restrict__ scores_out, int64_t bh, int i0,
                                               unsigned char *smem) {
    const int nb = prm.nb;
    const int nbp = (nb + 3) & ~3;
    float *sS = reinterpret_cast<float *>(smem);                  // [kRows][nbp]
    float *sQt = sS + kRows * nbp;                                // [D][kRows]
    uint32_t *sH = reinterpret_cast<uint32_t *>(sQt + D * kRows);  // [kWarps][kHistWords]
    uint32_t *sW = sH + kWarps * kHistWords;                      // [kWarps][kMaxWords]
    int *sE = reinterpret_cast<int *>(sW + kWarps * kMaxWords);   // [kWarps][kCand]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rows_here = min(kRows, nb - i0);

    // ---- phase 1
    for (int idx = tid; idx < kRows * D; idx += kThreads) {
        const int r = idx / D, d = idx % D;
        sQt[d * kRows + r] = (r < rows_here) ? __ldcg(qbar + (bh * nb + i0 + r) * D + d) : 0.f;
    }
    __syncthreads();
    const float *kt = kbar_t + bh * static_cast<int64_t>(D) * nbp;
    const uint64_t sc2 = f2_pack(prm.scale, prm.scale);
    for (int pc = tid; 2 * pc < nbp; pc += kThreads) {
        const int j = 2 * pc;  // columns j, j + 1 (pad columns past nb are zero)
        uint64_t acc[2][kRows / 2];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int q = 0; q < kRows / 2; ++q) acc[c][q] = 0ull;
        float2 kc[kPre], kn[kPre];
#pragma unroll
        for (int q = 0; q < kPre; ++q)
            kc[q] = __ldcg(reinterpret_cast<const float2 *>(kt + static_cast<int64_t>(q) * nbp + j));
#pragma unroll
        for (int d0 = 0; d0 < D; d0 += kPre) {
            if (d0 + kPre < D) {
#pragma unroll
                for (int q = 0; q < kPre; ++q)
                    kn[q] = __ldcg(reinterpret_cast<const float2 *>(
                        kt + static_cast<int64_t>(d0 + kPre + q) * nbp + j));
            }
#pragma unroll
            for (int q = 0; q < kPre; ++q) {
                const float4 *qv = reinterpret_cast<const float4 *>(sQt + (d0 + q) * kRows);
                const uint64_t k0 = f2_pack(kc[q].x, kc[q].x), k1 = f2_pack(kc[q].y, kc[q].y);
#pragma unroll
                for (int v = 0; v < kRows / 4; ++v) {
                    const float4 qq = qv[v];
                    const uint64_t qa = f2_pack(qq.x, qq.y), qb = f2_pack(qq.z, qq.w);
                    acc[0][2 * v] = f2_fma(qa, k0, acc[0][2 * v]);
                    acc[0][2 * v + 1] = f2_fma(qb, k0, acc[0][2 * v + 1]);
                    acc[1][2 * v] = f2_fma(qa, k1, acc[1][2 * v]);
                    acc[1][2 * v + 1] = f2_fma(qb, k1, acc[1][2 * v + 1]);
                }
            }
            if (d0 + kPre < D) {
#pragma unroll
                for (int q = 0; q < kPre; ++q) kc[q] = kn[q];
            }
        }
#pragma unroll
        for (int q = 0; q < kRows / 2; ++q) {
            const uint64_t a = f2_mul(acc[0][q], sc2), b = f2_mul(acc[1][q], sc2);
            *reinterpret_cast<float2 *>(sS + (2 * q) * nbp + j) = make_float2(f2_lo(a), f2_lo(b));
            *reinterpret_cast<float2 *>(sS + (2 * q + 1) * nbp + j) = make_float2(f2_hi(a), f2_hi(b));
        }
    }
    __syncthreads();  // scores complete

    if (scores_out != nullptr) {  // NABLA_DEBUG_SCORES: the rows as computed
        for (int idx = tid; idx < rows_here * nb; idx += kThreads) {
            const int r = idx / nb, j = idx % nb;
            scores_out[(bh * nb + i0 + r) * static_cast<int64_t>(nb) + j] = sS[r * nbp + j];
        }
    }

    // ---- phase 2: one warp per row
    const int words = (nb + 31) >> 5;
    const unsigned lt = (1u << lane) - 1u;
    uint32_t *hist = sH + warp * kHistWords;  // hi[256] | lo[256]
    uint32_t *sw = sW + warp * kMaxWords;
    int *ent = sE + warp * kCand;
    for (int r = warp; r < rows_here; r += kWarps) {
        const int i = i0 + r;
        const float *srow = sS + r * nbp;
        auto score = [&](int j) { return j < nb ? srow[j] : -INFINITY; };
        auto clear_hist = [&]() {
            uint4 *h4 = reinterpret_cast<uint4 *>(hist);
            for (int k = lane; k < kHistWords / 4; k += 32) h4[k] = make_uint4(0u, 0u, 0u, 0u);
        };

        // row maximum and minimum
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float mn[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
        for (int e0 = 0; e0 < words; e0 += 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = (e0 + u) * 32 + lane;
                if (j < nb) {
                    const float s = srow[j];
                    mx[u] = fmaxf(mx[u], s);
                    mn[u] = fminf(mn[u], s);
                }
            }
        }
        float smax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        float smin = fminf(fminf(mn[0], mn[1]), fminf(mn[2], mn[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
            smin = fminf(smin, __shfl_xor_sync(0xffffffffu, smin, o));
        }
        if (prm.mode == 1) {
            // logit threshold: keep the blocks within tau of the row's best
            for (int e = 0; e < words; ++e) {
                const float s = score(e * 32 + lane);
                const unsigned keep = __ballot_sync(0xffffffffu, s > -INFINITY &&
                                                                     __fsub_rn(smax, s) <= prm.tau);
                if (lane == 0) sw[e] = keep;
            }
            finish_row(prm, bh, i, sw, bits, row_idx, row_cnt);
            continue;
        }
        // bins over [0, span) of s_max - s; beyond 28 the masses are 0
        // (e^-28 * 2^40 < 1), so those blocks may share the last bin
        const float span = fminf(fmaxf(__fsub_rn(smax, smin), 0.0009765625f), 28.0f);
        const float g = __fdiv_rn(256.0f, span);

        // level 0: every block's mass into the bin of its key's top byte, and
        // the row total
        clear_hist();
        __syncwarp();
        double U = 0.0;
        for (int e0 = 0; e0 < words; e0 += 8) {
            float s[8];
            double u[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) s[q] = score((e0 + q) * 32 + lane);
#pragma unroll
            for (int q = 0; q < 8; ++q) u[q] = mass_of(s[q], smax);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                U += u[q];
                if (u[q] > 0.0) hist_add(hist, ykey(s[q], smax, g) >> 16, u[q]);
            }
        }
        U = warp_sum(U);
        const double thr = static_cast<double>(prm.p) * U;
        __syncwarp();

        // refine: at level L the cell is the blocks whose key has the L bytes
        // fixed so far; its bins are the key's next byte
        double before = 0.0;  // mass ranked above the cell
        uint32_t prefix = 0;  // key bytes fixed so far
        bool done = false;
        for (int lvl = 0; lvl < 3 && !done; ++lvl) {
            const int pshift = 24 - 8 * lvl, dshift = 16 - 8 * lvl;
            // scan of the cell's bins (8 per lane, in rank order)
            double hm[8], tot = 0.0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int b = lane * 8 + k;
                hm[k] = static_cast<double>(hist[b]) * 1048576.0 + static_cast<double>(hist[kBins + b]);
                tot += hm[k];
            }
            double incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const unsigned crossing = __ballot_sync(0xffffffffu, before + incl >= thr);
            if (crossing == 0u) {  // only a row with non-finite scores: keep it whole
                for (int e = lane; e < words; e += 32) sw[e] = 0xFFFFFFFFu;
                done = true;
                break;
            }
            const int owner = __ffs(crossing) - 1;
            int kk = 0;
            double c = before + incl - tot;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (c + hm[k] >= thr) break;
                c += hm[k];
                ++kk;
            }
            const uint32_t dig = static_cast<uint32_t>(__shfl_sync(0xffffffffu, lane * 8 + kk, owner));
            before = __shfl_sync(0xffffffffu, c, owner);
            __syncwarp();  // every lane has read the bins

            // one pass: cell blocks in lower bins are kept; those in the
            // crossing bin are the candidates (the first 64 listed)
            int m = 0;
            for (int e0 = 0; e0 < words; e0 += 4) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = e0 + q;
                    if (e < words) {
                        const float s = score(e * 32 + lane);
                        const uint32_t y = ykey(s, smax, g);
                        const bool member = s > -INFINITY && (lvl == 0 || (y >> pshift) == prefix);
                        const uint32_t b = (y >> dshift) & 255u;
                        const unsigned above = __ballot_sync(0xffffffffu, member && b < dig);
                        const bool cand = member && b == dig;
                        const unsigned bc = __ballot_sync(0xffffffffu, cand);
                        if (lane == 0) sw[e] = lvl == 0 ? above : (sw[e] | above);
                        if (cand) {
                            const int pos = m + __popc(bc & lt);
                            if (pos < kCand) ent[pos] = e * 32 + lane;
                        }
                        m += __popc(bc);
                    }
                }
            }
            if (m > kCand && lvl < 2) {
                // too many to rank at once: histogram the crossing bin's blocks
                // by the key's next byte for the next level
                const uint32_t cell = (prefix << 8) | dig;
                clear_hist();
                __syncwarp();
                for (int e = 0; e < words; ++e) {
                    const float s = score(e * 32 + lane);
                    const uint32_t y = ykey(s, smax, g);
                    if (s > -INFINITY && (y >> dshift) == cell) {
                        const double u = mass_of(s, smax);
                        if (u > 0.0) hist_add(hist, (y >> (dshift - 8)) & 255u, u);
                    }
                }
            }
            prefix = (prefix << 8) | dig;
            __syncwarp();
            if (m <= kCand) {
                // exact rank among the candidates: the last kept block is the
                // highest-ranked candidate whose inclusive mass (candidates
                // ranked at or above it) reaches thr - before
                int jc[2];
                double uc[2];
                uint64_t Kc[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int slot = h * 32 + lane;
                    jc[h] = slot < m ? ent[slot] : 0;
                    const float s = slot < m ? srow[jc[h]] : -INFINITY;
                    uc[h] = slot < m ? mass_of(s, smax) : 0.0;
                    Kc[h] = slot < m ? rank_key(s, jc[h]) : 0ull;
                }
                double S[2] = {0.0, 0.0};
                for (int t = 0; t < m; ++t) {
                    const uint64_t Kt = __shfl_sync(0xffffffffu, t < 32 ? Kc[0] : Kc[1], t & 31);
                    const double ut = __shfl_sync(0xffffffffu, t < 32 ? uc[0] : uc[1], t & 31);
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        if (Kt >= Kc[h]) S[h] += ut;
                }
                uint64_t best = 0ull;
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if (h * 32 + lane < m && before + S[h] >= thr) best = max(best, Kc[h]);
                const uint64_t kstar = warp_max_u64(best);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if (h * 32 + lane < m && Kc[h] >= kstar)
                        atomicOr(sw + (jc[h] >> 5), 1u << (jc[h] & 31));
                done = true;
            }
        }
        if (!done) {
            // more than 64 blocks share all three key bytes: take the cell's
            // score groups from the top (one score per group, so one mass);
            // the group that reaches thr keeps its lowest indices first
            uint64_t bound = 1ull << 32;  // groups at or above this order key are taken
            for (int guard = 0; guard < nb; ++guard) {
                uint32_t okm = 0u;
                bool any = false;
                for (int e = 0; e < words; ++e) {
                    const float s = score(e * 32 + lane);
                    const uint32_t ok = order_key(s);
                    if (s > -INFINITY && ykey(s, smax, g) == prefix && ok < bound) {
                        okm = max(okm, ok);
                        any = true;
                    }
                }
                if (__ballot_sync(0xffffffffu, any) == 0u) break;
                const uint32_t tau = __reduce_max_sync(0xffffffffu, any ? okm : 0u);
                // the group's score (order_key inverted) and its common mass
                const float sg = __uint_as_float((tau & 0x80000000u) ? (tau & 0x7FFFFFFFu) : ~tau);
                const double ug = mass_of(sg, smax);
                int gn = 0;
                for (int e = 0; e < words; ++e) {
                    const float s = score(e * 32 + lane);
                    gn += __popc(__ballot_sync(0xffffffffu, s > -INFINITY &&
                                                                ykey(s, smax, g) == prefix &&
                                                                order_key(s) == tau));
                }
                const bool last = before + static_cast<double>(gn) * ug >= thr;
                int t = gn;  // members of the group kept, lowest index first
                if (last) {
                    t = static_cast<int>(ceil((thr - before) / ug));
                    while (t > 1 && before + static_cast<double>(t - 1) * ug >= thr) --t;
                    while (t < gn && before + static_cast<double>(t) * ug < thr) ++t;
                }
                int seen = 0;
                for (int e = 0; e < words; ++e) {
                    const float s = score(e * 32 + lane);
                    const bool in = s > -INFINITY && ykey(s, smax, g) == prefix && order_key(s) == tau;
                    const unsigned b = __ballot_sync(0xffffffffu, in);
                    const unsigned kb = __ballot_sync(0xffffffffu, in && seen + __popc(b & lt) < t);
                    if (lane == 0) sw[e] |= kb;
                    seen += __popc(b);
                }
                before += static_cast<double>(gn) * ug;
                if (last) break;
                bound = tau;
            }
        }
        __syncwarp();

        finish_row(prm, bh, i, sw, bits, row_idx, row_cnt);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3)
    score_cut_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar_t,
                     CutParams prm, uint32_t *__restrict__ bits, uint16_t *__restrict__ row_idx,
                     int32_t *__restrict__ row_cnt, float *__restrict__ scores_out) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int tiles = (prm.nb + kRows - 1) / kRows;
    score_cut_tile<D>(qbar, kbar_t, prm, bits, row_idx, row_cnt, scores_out, blockIdx.x / tiles,
                      static_cast<int>(blockIdx.x % tiles) * kRows, smem);
}

// ---------------------------------------------------------------------------
// Persistent front end: the pooling (or flattening + pooling) tiles and the
// score/cut tiles of every head in one launch, so that the HBM-bound pooling
// of head h + 1 runs beside the issue-bound scores and cut of head h.  CTAs
// take tasks in order from a counter: the pooling tiles of head 0, then for
// h = 1 .. BH the pooling tiles of head h (while h < BH) followed by the
// score/cut tiles of head h - 1.  A score/cut tile waits until its head's
// pooling tiles have all finished (a per-head counter; every pooling tile it
// needs was taken earlier by a running CTA that never waits, so the wait
// always ends); the wait is bounded (1 s of %globaltimer), after which the
// status word records a timeout and the remaining score/cut tiles are
// skipped.  ctr[0] = next task, ctr[1 + bh] = finished pooling tiles of head
// bh, all zero at launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <int D, bool kGrid>
__global__ void __launch_bounds__(kThreads, 3)
    front_kernel(const __nv_bfloat16 *__restrict__ q_grid, const __nv_bfloat16 *__restrict__ k_grid,
                 const __nv_bfloat16 *q, const __nv_bfloat16 *k, float *qbar, float *kbar_t,
                 CutParams prm, uint32_t *__restrict__ bits, uint16_t *__restrict__ row_idx,
                 int32_t *__restrict__ row_cnt, float *__restrict__ scores_out, int *ctr,
                 int *status, int64_t BH, int H, int W) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_task, s_go;
    constexpr int BPC = 256 / (D / 8);
    const int nb = prm.nb;
    const int tiles = (nb + BPC - 1) / BPC;
    const int P = 2 * tiles;                    // pooling tiles per head (Q and K)
    const int S = (nb + kRows - 1) / kRows;     // score/cut tiles per head
    const int64_t total = BH * static_cast<int64_t>(P + S);
    float(*tile)[D + 1] = reinterpret_cast<float(*)[D + 1]>(smem);
    for (;;) {
        __syncthreads();  // the previous task is done with shared memory
        if (threadIdx.x == 0) s_task = atomicAdd(ctr, 1);
        __syncthreads();
        const int64_t t = s_task;
        if (t >= total) break;
        // decode: [P pool(0)] [P pool(1), S score(0)] ... [P pool(BH-1), S score(BH-2)] [S score(BH-1)]
        bool pool;
        int64_t bh;
        int idx;
        if (t < P) {
            pool = true, bh = 0, idx = static_cast<int>(t);
        } else {
            const int64_t u = t - P, blk = u / (P + S);
            const int r = static_cast<int>(u % (P + S));
            if (blk + 1 < BH) {
                pool = r < P;
                bh = pool ? blk + 1 : blk;
                idx = pool ? r : r - P;
            } else {
                pool = false, bh = BH - 1, idx = static_cast<int>(u - (BH - 1) * (P + S));
            }
        }
        if (pool) {
            const int64_t cta = (idx / tiles) * BH * tiles + bh * tiles + idx % tiles;
            if (kGrid)
                flatten_pool_tile<D>(q_grid, k_grid, const_cast<__nv_bfloat16 *>(q),
                                     const_cast<__nv_bfloat16 *>(k), qbar, kbar_t, BH, nb, H, W,
                                     cta, tile);
            else
                pool_tile<D>(q, k, qbar, kbar_t, BH, nb, cta, tile);
            __threadfence();  // this thread's pooled means, visible GPU-wide
            __syncthreads();
            if (threadIdx.x == 0) atomicAdd(ctr + 1 + bh, 1);
        } else {
            if (threadIdx.x == 0) {
                // the test aid NABLA_DEBUG_TIMEOUT waits for one pooling tile
                // too many, with a 1 ms limit: the wait must run out
                const bool test_wait = (prm.flags & 0x100u) != 0;
                const int need = test_wait ? P + 1 : P;
                const uint64_t limit = test_wait ? 1000000ull : 1000000000ull;
                int go = *reinterpret_cast<volatile int *>(status) == kDevOk;
                if (go && ld_acquire_gpu(ctr + 1 + bh) < need) {
                    const uint64_t t0 = global_ns();
                    for (int n = 0; ld_acquire_gpu(ctr + 1 + bh) < need; ++n) {
                        if (global_ns() - t0 > limit) {  // give up
                            atomicExch(status, kDevTimeout);
                            go = 0;
                            break;
                        }
                        if (n > 64) __nanosleep(128);
                    }
                }
                s_go = go;
            }
            __syncthreads();
            if (s_go)
                score_cut_tile<D>(qbar, kbar_t, prm, bits, row_idx, row_cnt, scores_out, bh,
                                  idx * kRows, smem);
        }
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
// DynamicRad static-ratio mask ("DynamicRad: Content-Adaptive Sparse Attention
// for Long Video Diffusion", section 2.A, Static-Ratio mode): content-free.
// Query block i = (t_i, q) keeps, in every frame t, the k(|t - t_i|) patches
// nearest to its patch q (squared distance in patch units, then block index).
// One CTA per (bh, patch position q): the patch ranks around q and the counts
// k(dt) are computed once into shared memory, then one warp per frame t_i
// builds the row of block (t_i, q).
// ---------------------------------------------------------------------------
struct RatioParams {
    double gamma, lambda;
};

__global__ void __launch_bounds__(256) ratio_kernel(CutParams prm, RatioParams rp,
                                                    uint32_t *__restrict__ bits,
                                                    uint16_t *__restrict__ row_idx,
                                                    int32_t *__restrict__ row_cnt) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int nb = prm.nb, T = prm.T, Wp = prm.Wp, HW = prm.Hp * prm.Wp;
    const int words = (nb + 31) >> 5;
    uint32_t *sW = reinterpret_cast<uint32_t *>(smem);            // [8][kMaxWords]
    int *rank = reinterpret_cast<int *>(sW + 8 * kMaxWords);        // [HW]
    int *kcnt = rank + HW;                                          // [T]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.x / HW;
    const int q = static_cast<int>(blockIdx.x % HW);
    const int qh = q / Wp, qw = q % Wp;
    // (with one frame every row keeps its whole frame: no ranks needed)
    for (int p = tid; T > 1 && p < HW; p += blockDim.x) {
        const int dh = p / Wp - qh, dw = p % Wp - qw, dp = dh * dh + dw * dw;
        int r = 0;
        for (int p2 = 0; p2 < HW; ++p2) {
            const int eh = p2 / Wp - qh, ew = p2 % Wp - qw, d2 = eh * eh + ew * ew;
            r += (d2 < dp || (d2 == dp && p2 < p)) ? 1 : 0;
        }
        rank[p] = r;
    }
    for (int dt = tid; dt < T; dt += blockDim.x) {
        double g = 1.0;
        for (int n = 0; n < dt; ++n) g = __dmul_rn(g, rp.gamma);  // gamma^dt, dt factors
        const double r = fmin(1.0, fmax(rp.lambda, g));
        kcnt[dt] = static_cast<int>(fmin(ceil(__dmul_rn(r, static_cast<double>(HW))),
                                         static_cast<double>(HW)));
    }
    __syncthreads();
    uint32_t *sw = sW + warp * kMaxWords;
    for (int ti = warp; ti < T; ti += 8) {
        const int i = ti * HW + q;
        for (int e = 0; e < words; ++e) {
            const int j = e * 32 + lane;
            bool keep = false;
            if (j < nb) {
                const int tj = j / HW, dt = tj > ti ? tj - ti : ti - tj;
                keep = kcnt[dt] >= HW || rank[j - tj * HW] < kcnt[dt];
            }
            const unsigned b = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) sw[e] = b;
        }
        finish_row(prm, bh, i, sw, bits, row_idx, row_cnt);
    }
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
    return sizeof(float) * (nabla::kRows * nbp + static_cast<size_t>(D) * nabla::kRows) +
           sizeof(uint32_t) * nabla::kWarps * (nabla::kHistWords + nabla::kMaxWords) +
           sizeof(int) * nabla::kWarps * nabla::kCand;
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

template <int D, bool kGrid>
static cudaError_t launch_front(const void *q_grid, const void *k_grid, const void *q,
                                const void *k, float *qbar, float *kbar_t, nabla::CutParams prm,
                                uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                                float *scores, int *ctr, int *status, int64_t BH, int H, int W,
                                cudaStream_t stream) {
    using namespace nabla;
    auto kern = front_kernel<D, kGrid>;
    const size_t smem = nabla_score_cut_smem(prm.nb, D);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 0, per_sm = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return err;
    if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) !=
        cudaSuccess)
        return err;
    const int bpc = 256 / (D / 8);
    const int64_t tasks =
        BH * (2 * ((prm.nb + bpc - 1) / bpc) + (prm.nb + kRows - 1) / kRows);
    const int64_t grid = std::min<int64_t>(tasks, static_cast<int64_t>(sms) * std::max(per_sm, 1));
    if ((err = cudaMemsetAsync(ctr, 0, sizeof(int) * (1 + BH), stream)) != cudaSuccess) return err;
    kern<<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(q_grid), static_cast<const __nv_bfloat16 *>(k_grid),
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), qbar, kbar_t,
        prm, bits, row_idx, row_cnt, scores, ctr, status, BH, H, W);
    return cudaGetLastError();
}

// q_grid/k_grid non-null: q and k are in grid order; flatten them into q/k
// (then outputs) in the same pass as the pooling.  scores non-null: also
// write the pooled scores [BH, nb, nb] (only when the mask depends on them).
// ctr non-null with grid-order inputs (1 + BH ints of device memory, cleared
// here): the flattening + pooling and the scores and cut run in one
// persistent launch; otherwise as a pooling launch followed by a score/cut
// launch.
cudaError_t nabla_launch_build_mask(int64_t BH, int nb, int D, int T, int Hp, int Wp, float p,
                                    float scale, int wt, int wh, int ww, unsigned flags,
                                    const void *q, const void *k, float *qbar, float *kbar_t,
                                    uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                                    uint16_t *col_idx, int32_t *col_cnt, float *scores,
                                    cudaStream_t stream, const void *q_grid, const void *k_grid,
                                    int *ctr, int *status) {
    using namespace nabla;
    CutParams prm{nb, T, Hp, Wp, wt, wh, ww, flags, p, scale, 0, 0.f};
    const bool score_free = p <= 0.0f || p >= 1.0f || (flags & 2u);
    if (ctr != nullptr && q_grid != nullptr && !score_free) {
        // flattening + pooling (HBM-bound, 2 x 2 bytes per element moved) beside
        // the scores and cut in one persistent launch.  (From already
        // flattened inputs the pooling is too short to gain from it: measured
        // no faster, so that case keeps the two launches below.)
        cudaError_t err =
            D == 128 ? launch_front<128, true>(q_grid, k_grid, q, k, qbar, kbar_t, prm, bits,
                                               row_idx, row_cnt, scores, ctr, status, BH, Hp * 8,
                                               Wp * 8, stream)
                     : launch_front<64, true>(q_grid, k_grid, q, k, qbar, kbar_t, prm, bits,
                                              row_idx, row_cnt, scores, ctr, status, BH, Hp * 8,
                                              Wp * 8, stream);
        if (err != cudaSuccess) return err;
        if (col_idx) {
            const int words = (nb + 31) / 32;
            col_lists_kernel<<<static_cast<unsigned>(BH * words), kColWarps * 32, 0, stream>>>(
                bits, col_idx, col_cnt, nb);
            err = cudaGetLastError();
        }
        return err;
    }
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
    if (score_free) {
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

// DynamicRad-style masks (mode 0: static ratio, mode 1: logit threshold) in
// the same list format; the threshold mode pools and scores like the NABLA
// path.
cudaError_t nabla_launch_build_mask_dr(int64_t BH, int nb, int D, int T, int Hp, int Wp, int mode,
                                       double gamma, double lambda, float tau, float scale, int wt,
                                       int wh, int ww, unsigned flags, const void *q,
                                       const void *k, float *qbar, float *kbar_t, uint32_t *bits,
                                       uint16_t *row_idx, int32_t *row_cnt, uint16_t *col_idx,
                                       int32_t *col_cnt, float *scores, cudaStream_t stream) {
    using namespace nabla;
    CutParams prm{nb, T, Hp, Wp, wt, wh, ww, flags, 1.0f, scale, mode, tau};
    cudaError_t err = cudaSuccess;
    const int words = (nb + 31) / 32;
    const dim3 col_grid(static_cast<unsigned>(BH * words));
    if (flags & 2u) {  // the full window: every block
        const int64_t rows = BH * nb;
        sta_emit_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, stream>>>(
            prm, rows, bits, row_idx, row_cnt);
    } else if (mode == 0) {
        const int HW = Hp * Wp;
        const size_t smem = sizeof(uint32_t) * 8 * kMaxWords + sizeof(int) * (HW + T);
        ratio_kernel<<<static_cast<unsigned>(BH * HW), 256, smem, stream>>>(
            prm, RatioParams{gamma, lambda}, bits, row_idx, row_cnt);
    } else {
        const int bpc = 256 / (D / 8);
        const int64_t tiles = (nb + bpc - 1) / bpc;
        const dim3 pool_grid(static_cast<unsigned>(2 * BH * tiles));
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
        const size_t smem = nabla_score_cut_smem(nb, D);
        const dim3 grid(static_cast<unsigned>(BH * ((nb + kRows - 1) / kRows)));
        err = D == 128 ? launch_score_cut<128>(grid, smem, qbar, kbar_t, prm, bits, row_idx,
                                               row_cnt, scores, stream)
                       : launch_score_cut<64>(grid, smem, qbar, kbar_t, prm, bits, row_idx,
                                              row_cnt, scores, stream);
        if (err != cudaSuccess) return err;
    }
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (col_idx) {
        col_lists_kernel<<<col_grid, kColWarps * 32, 0, stream>>>(bits, col_idx, col_cnt, nb);
        err = cudaGetLastError();
    }
    return err;
}
