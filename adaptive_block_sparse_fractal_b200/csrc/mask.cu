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
//                      per row (one warp, values in registers): weights
//                      exp(s - max) in float64, integer mass floor(w * 2^40),
//                      a bitwise bisection over the 48-bit key (score bits,
//                      then inverted block index, only when scores tie) for
//                      the last block of the shortest descending prefix whose
//                      mass reaches p * total, and the OR with the STA window
//                      and the diagonal.  Writes the bit row and the ascending
//                      row list.
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
            if (i0 + b < nb) kbar_t[(bh * D + d) * nbp + i0 + b] = tile[b][d];
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
            if (i0 + b < nb) kbar_t[(bh * D + d) * nbp + i0 + b] = tile[b][d];
        }
    }
}

// ---------------------------------------------------------------------------
// scores + CDF cut + STA + lists
// ---------------------------------------------------------------------------
constexpr int kRows = 16;    // query blocks per CTA
constexpr int kCols = 256;   // key blocks per score tile
constexpr int kDc = 32;      // features per staged K-bar slice
constexpr int kThreads = 256;

struct CutParams {
    int nb, Hp, Wp, wt, wh, ww;
    unsigned flags;
    float p, scale;
};

__device__ __forceinline__ uint32_t order_key(float s) {
    uint32_t b = __float_as_uint(s);
    if (b == 0x80000000u) b = 0u;  // -0 ranks with +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Integer mass floor(exp(s - smax) * 2^40), held in a double (exact: an
// integer <= 2^40; sums of up to 2^13 of them stay below 2^53, so every sum
// below is exact whatever the order of the additions).
__device__ __forceinline__ double mass_of(float s, float smax) {
    const double w = exp(static_cast<double>(s) - static_cast<double>(smax));
    return trunc(w * 1099511627776.0);  // * 2^40 is an exact scaling
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// (frame, patch row, patch column) of block j, advanced by a fixed stride
// without integer division (the emit loops visit j = lane, lane + 32, ...).
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

// One warp per query row.  E = elements per lane (nb <= 32 * E).
template <int D, int E>
__global__ void __launch_bounds__(kThreads, 1)
    score_cut_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar_t,
                     CutParams prm, uint32_t *__restrict__ bits, uint16_t *__restrict__ row_idx,
                     int32_t *__restrict__ row_cnt) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int nb = prm.nb;
    const int nbp = (nb + 3) & ~3;
    float *sS = reinterpret_cast<float *>(smem);                       // [kRows][nbp]
    float *sQt = reinterpret_cast<float *>(smem + sizeof(float) * kRows * nbp);  // [D][kRows]
    float *sKt = sQt + D * kRows;                                      // [2][kDc][kCols]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tiles = (nb + kRows - 1) / kRows;
    const int64_t bh = blockIdx.x / tiles;
    const int i0 = (blockIdx.x % tiles) * kRows;

    // ---- phase 1: scores s[r][j] = (fma chain over d of qbar_i . kbar_j) * scale
    // K-bar slices [kDc features][kCols blocks] stream through a double buffer
    // with cp.async; the accumulation per output still runs d = 0, 1, ... D-1.
    for (int idx = tid; idx < kRows * D; idx += kThreads) {
        const int r = idx / D, d = idx % D;
        sQt[d * kRows + r] = (i0 + r < nb) ? qbar[(bh * nb + i0 + r) * D + d] : 0.f;
    }
    const int cg = tid % 64;  // 4 consecutive columns
    const int rg = tid / 64;  // 4 consecutive rows
    const float *kt = kbar_t + bh * static_cast<int64_t>(D) * nbp;
    constexpr int DCH = D / kDc;  // feature slices per column tile
    const int nstage = ((nb + kCols - 1) / kCols) * DCH;
    auto issue = [&](int st) {
        const int j0 = (st / DCH) * kCols, d0 = (st % DCH) * kDc;
        float *dst = sKt + (st & 1) * (kDc * kCols);
        // kDc rows of kCols floats = kDc * kCols / 4 chunks of 16 bytes
        for (int c = tid; c < kDc * kCols / 4; c += kThreads) {
            const int d = c / (kCols / 4), j = (c % (kCols / 4)) * 4;
            float *sd = dst + d * kCols + j;
            if (j0 + j < nbp) {
                cp_async16(smem_addr(sd), kt + static_cast<int64_t>(d0 + d) * nbp + j0 + j);
            } else {
                sd[0] = sd[1] = sd[2] = sd[3] = 0.f;
            }
        }
        cp_async_commit();
    };
    float acc[4][4];
    issue(0);
    for (int st = 0; st < nstage; ++st) {
        if (st + 1 < nstage) {
            issue(st + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int j0 = (st / DCH) * kCols, d0 = (st % DCH) * kDc;
        if (d0 == 0) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
        }
        const float *sk = sKt + (st & 1) * (kDc * kCols);
#pragma unroll 8
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
        __syncthreads();
    }

    // ---- phase 2: one warp per row; keys and masses in registers
    const int words = (nb + 31) >> 5;
    const bool keep_all = prm.p >= 1.0f;
    const bool keep_none = prm.p <= 0.0f;
    for (int r = warp; r < kRows; r += kThreads / 32) {
        const int i = i0 + r;
        if (i >= nb) break;
        const float *srow = sS + r * nbp;
        uint64_t cstar = 0;  // composite key (score key, 0xFFFF - j) of the last kept block
        if (!keep_all && !keep_none) {
            uint32_t kv[E];
            double wv[E];
            float smax = -INFINITY;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = lane + 32 * e;
                if (j < nb) smax = fmaxf(smax, srow[j]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
            double U = 0.0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = lane + 32 * e;
                const float sv = j < nb ? srow[j] : 0.f;
                kv[e] = j < nb ? order_key(sv) : 0u;
                wv[e] = j < nb ? mass_of(sv, smax) : 0.0;
                U += wv[e];
            }
            U = warp_sum(U);
            const double thr = static_cast<double>(prm.p) * U;
            // largest score key tau with mass(key >= tau) >= thr
            uint32_t tau = 0;
            for (int b = 31; b >= 0; --b) {
                const uint32_t cand = tau | (1u << b);
                double m0 = 0.0, m1 = 0.0;
#pragma unroll
                for (int e = 0; e < E; e += 2) {
                    if (kv[e] >= cand) m0 += wv[e];
                    if (e + 1 < E && kv[e + 1] >= cand) m1 += wv[e + 1];
                }
                if (warp_sum(m0 + m1) >= thr) tau = cand;
            }
            // blocks sharing the score key tau are taken in ascending index
            int nt = 0, jt = -1;
            double above = 0.0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = lane + 32 * e;
                if (j < nb && kv[e] == tau) {
                    ++nt;
                    jt = j;
                }
                if (kv[e] > tau) above += wv[e];
            }
            for (int o = 16; o > 0; o >>= 1) {
                nt += __shfl_xor_sync(0xffffffffu, nt, o);
                jt = max(jt, __shfl_xor_sync(0xffffffffu, jt, o));
            }
            uint32_t xs;  // 0xFFFF - index of the last kept block
            if (nt == 1) {
                xs = 0xFFFFu - static_cast<uint32_t>(jt);
            } else {
                above = warp_sum(above);
                xs = 0;
                for (int b = 15; b >= 0; --b) {
                    const uint32_t cand = xs | (1u << b);
                    double m = 0.0;
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int j = lane + 32 * e;
                        if (j < nb && kv[e] == tau && (0xFFFFu - j) >= cand) m += wv[e];
                    }
                    if (above + warp_sum(m) >= thr) xs = cand;
                }
            }
            cstar = (static_cast<uint64_t>(tau) << 16) | xs;
        }
        // emit: bit row + ascending list
        const BlockCoord ci(i, prm.Hp, prm.Wp);
        BlockCoord cj(lane, prm.Hp, prm.Wp);
        int cnt = 0;
        uint16_t *lst = row_idx + (bh * nb + i) * static_cast<int64_t>(nb);
        for (int w = 0; w < words; ++w, cj.advance(32, prm.Hp, prm.Wp)) {
            const int j = w * 32 + lane;
            bool m = false;
            if (j < nb) {
                if (keep_all) {
                    m = true;
                } else if (!keep_none) {
                    const uint64_t key = (static_cast<uint64_t>(order_key(srow[j])) << 16) |
                                         static_cast<uint64_t>(0xFFFFu - j);
                    m = key >= cstar;
                }
                m = m || (j == i) || (prm.flags & 2u);
                if (!m && !(prm.flags & 1u)) m = in_window(ci, cj, prm);
            }
            const unsigned ball = __ballot_sync(0xffffffffu, m);
            if (lane == 0) bits[(bh * nb + i) * words + w] = ball;
            if (m) lst[cnt + __popc(ball & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
            cnt += __popc(ball);
        }
        if (lane == 0) row_cnt[bh * nb + i] = cnt;
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
// column lists: transpose of the bit rows.  One warp per (bh, 32-column word).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) col_lists_kernel(const uint32_t *__restrict__ bits,
                                                        uint16_t *__restrict__ col_idx,
                                                        int32_t *__restrict__ col_cnt,
                                                        int64_t BH, int nb) {
    const int words = (nb + 31) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (gw >= BH * words) return;
    const int64_t bh = gw / words;
    const int w = static_cast<int>(gw % words);
    const int j = w * 32 + lane;  // this lane's column
    int cnt = 0;
    uint16_t *lst = col_idx + (bh * nb + (j < nb ? j : 0)) * static_cast<int64_t>(nb);
    for (int i0 = 0; i0 < nb; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t word = (i < nb) ? bits[(bh * nb + i) * words + w] : 0u;
        uint32_t mine = 0;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const uint32_t col = __ballot_sync(0xffffffffu, (word >> c) & 1u);
            if (lane == c) mine = col;
        }
        if (j < nb) {
            while (mine) {
                const int b = __ffs(mine) - 1;
                mine &= mine - 1;
                lst[cnt++] = static_cast<uint16_t>(i0 + b);
            }
        }
    }
    if (j < nb) col_cnt[bh * nb + j] = cnt;
}

}  // namespace nabla

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
size_t nabla_score_cut_smem(int nb, int D) {
    const size_t nbp = (static_cast<size_t>(nb) + 3) & ~static_cast<size_t>(3);
    const size_t phase1 = sizeof(float) * (static_cast<size_t>(D) * nabla::kRows +
                                           2 * nabla::kDc * nabla::kCols);
    return sizeof(float) * nabla::kRows * nbp + phase1;
}

template <int D, int E>
static cudaError_t launch_score_cut(dim3 grid, size_t smem, const float *qbar,
                                    const float *kbar_t, nabla::CutParams prm, uint32_t *bits,
                                    uint16_t *row_idx, int32_t *row_cnt, cudaStream_t stream) {
    cudaError_t err = cudaFuncSetAttribute(nabla::score_cut_kernel<D, E>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    nabla::score_cut_kernel<D, E><<<grid, nabla::kThreads, smem, stream>>>(qbar, kbar_t, prm, bits,
                                                                           row_idx, row_cnt);
    return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_score_cut(dim3 grid, size_t smem, const float *qbar,
                                      const float *kbar_t, nabla::CutParams prm, uint32_t *bits,
                                      uint16_t *row_idx, int32_t *row_cnt, cudaStream_t stream) {
    const int e = (prm.nb + 31) / 32;
#define NABLA_SC(EV)                                                                          \
    if (e <= EV)                                                                              \
        return launch_score_cut<D, EV>(grid, smem, qbar, kbar_t, prm, bits, row_idx, row_cnt, \
                                       stream);
    NABLA_SC(1) NABLA_SC(4) NABLA_SC(16) NABLA_SC(40) NABLA_SC(48) NABLA_SC(64)
#undef NABLA_SC
    return cudaErrorInvalidValue;
}

// q_grid/k_grid non-null: q and k are in grid order; flatten them into q/k
// (then outputs) in the same pass as the pooling.
cudaError_t nabla_launch_build_mask(int64_t BH, int nb, int D, int Hp, int Wp, float p,
                                    float scale, int wt, int wh, int ww, unsigned flags,
                                    const void *q, const void *k, float *qbar, float *kbar_t,
                                    uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                                    uint16_t *col_idx, int32_t *col_cnt, cudaStream_t stream,
                                    const void *q_grid, const void *k_grid) {
    using namespace nabla;
    CutParams prm{nb, Hp, Wp, wt, wh, ww, flags, p, scale};
    cudaError_t err;
    const bool from_grid = q_grid != nullptr;
    const int bpc = 256 / (D / 8);
    const int64_t tiles = (nb + bpc - 1) / bpc;
    const dim3 pool_grid(static_cast<unsigned>(2 * BH * tiles));
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
            const int64_t warps = BH * ((nb + 31) / 32);
            col_lists_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(
                bits, col_idx, col_cnt, BH, nb);
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
    err = D == 128 ? dispatch_score_cut<128>(grid, smem, qbar, kbar_t, prm, bits, row_idx, row_cnt,
                                             stream)
                   : dispatch_score_cut<64>(grid, smem, qbar, kbar_t, prm, bits, row_idx, row_cnt,
                                            stream);
    if (err != cudaSuccess) return err;
    if (col_idx) {
        const int64_t warps = BH * ((nb + 31) / 32);
        col_lists_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(
            bits, col_idx, col_cnt, BH, nb);
        err = cudaGetLastError();
    }
    return err;
}
