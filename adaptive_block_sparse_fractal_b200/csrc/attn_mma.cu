// Block-sparse flash attention over the NABLA block mask, warp-level
// mma.sync (bf16 m16n8k16, fp32 accumulate) version.
//
// "NABLA: Neighborhood Adaptive Block-Level Attention", section 手法: NABLA,
// bullet "拡張": attention is computed for the kept 64 x 64 blocks only.
//
//   fwd_kernel      one CTA per (bh, query block i); 4 warps x 16 queries;
//                   walks row list i with double-buffered cp.async K/V tiles;
//                   online softmax in registers (base-2 exponent).
//   bwd_pre_kernel  D_n = dO_n . O_n.
//   bwd_dkdv_kernel one CTA per (bh, key block j), walks column list j:
//                   S^T = K Q^T, P^T = exp(S^T - lse), dV += P^T dO,
//                   dP^T = V dO^T, dS^T = P^T (dP^T - D), dK += dS^T Q.
//   bwd_dq_kernel   one CTA per (bh, query block i), walks row list i:
//                   dQ += (P (dO V^T - D)) K.
// No atomics: every output tile has exactly one writer.
#include "common.cuh"

namespace nabla {
namespace mma {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// A fragment (16 rows x 16 k) from a swizzled [rows][CH chunks] tile.
template <int CH>
__device__ __forceinline__ void lda(uint32_t tile, int row0, int kk, uint32_t *a) {
    const int lane = threadIdx.x & 31;
    const int r = row0 + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int c = 2 * kk + (lane >> 4);
    ldsm_x4(tile + swz<CH>(r, c), a[0], a[1], a[2], a[3]);
}
// B fragments of two n-tiles (n0.., n0+8..) from a tile stored [n][k].
template <int CH>
__device__ __forceinline__ void ldb_nk(uint32_t tile, int n0, int kk, uint32_t *b) {
    const int lane = threadIdx.x & 31;
    const int r = n0 + (lane & 7) + 8 * (lane >> 4);
    const int c = 2 * kk + ((lane >> 3) & 1);
    ldsm_x4(tile + swz<CH>(r, c), b[0], b[1], b[2], b[3]);
}
// B fragments of two n-tiles (chunks c0, c0+1) from a tile stored [k][n].
template <int CH>
__device__ __forceinline__ void ldb_kn(uint32_t tile, int k0, int c0, uint32_t *b) {
    const int lane = threadIdx.x & 31;
    const int r = k0 + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int c = c0 + (lane >> 4);
    ldsm_x4_t(tile + swz<CH>(r, c), b[0], b[1], b[2], b[3]);
}
// Async copy of a [64][D] bf16 tile (row stride D) into a swizzled tile.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t tile, const __nv_bfloat16 *g, int nthreads) {
    constexpr int CH = D / 8;
    for (int idx = threadIdx.x; idx < kBlk * CH; idx += nthreads) {
        const int r = idx / CH, c = idx % CH;
        cp_async16(tile + swz<CH>(r, c), g + static_cast<int64_t>(r) * D + c * 8);
    }
}

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) fwd_kernel(const __nv_bfloat16 *__restrict__ q,
                                                  const __nv_bfloat16 *__restrict__ k,
                                                  const __nv_bfloat16 *__restrict__ v,
                                                  const uint16_t *__restrict__ row_idx,
                                                  const int32_t *__restrict__ row_cnt,
                                                  __nv_bfloat16 *__restrict__ o,
                                                  float *__restrict__ lse, int nb, float scale) {
    constexpr int CH = D / 8;
    constexpr int TILE = kBlk * D * 2;
    constexpr int KT = D / 16;  // k-steps over features
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t sQ = smem_addr(smem);
    const uint32_t sK0 = sQ + TILE, sV0 = sQ + 3 * TILE;  // K: [2], V: [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = blockIdx.x / nb;
    const int i = blockIdx.x % nb;
    const int64_t N = static_cast<int64_t>(nb) * kBlk;
    const int cnt = row_cnt[bh * nb + i];
    const uint16_t *lst = row_idx + (bh * nb + i) * static_cast<int64_t>(nb);
    const __nv_bfloat16 *kh = k + bh * N * D, *vh = v + bh * N * D;
    const float sl = scale * kLog2e;

    float oacc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    load_tile<D>(sQ, q + (bh * N + static_cast<int64_t>(i) * kBlk) * D, 128);
    if (cnt > 0) {
        const int j = lst[0];
        load_tile<D>(sK0, kh + static_cast<int64_t>(j) * kBlk * D, 128);
        load_tile<D>(sV0, vh + static_cast<int64_t>(j) * kBlk * D, 128);
    }
    cp_async_commit();

    uint32_t qf[KT][4];
    for (int e = 0; e < cnt; ++e) {
        const int buf = e & 1;
        if (e + 1 < cnt) {
            const int j = lst[e + 1];
            load_tile<D>(sK0 + (buf ^ 1) * TILE, kh + static_cast<int64_t>(j) * kBlk * D, 128);
            load_tile<D>(sV0 + (buf ^ 1) * TILE, vh + static_cast<int64_t>(j) * kBlk * D, 128);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (e == 0) {
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) lda<CH>(sQ, warp * 16, kk, qf[kk]);
        }
        const uint32_t sK = sK0 + buf * TILE, sV = sV0 + buf * TILE;
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b[4];
                ldb_nk<CH>(sK, np * 16, kk, b);
                mma_bf16(s[2 * np], qf[kk], b[0], b[1]);
                mma_bf16(s[2 * np + 1], qf[kk], b[2], b[3]);
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
            mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
        }
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0 * sl), mn1 = fmaxf(m1, mx1 * sl);
        const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        float ps0 = 0.f, ps1 = 0.f;
        uint32_t pf[4][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const float p0 = fast_exp2(fmaf(s[n][0], sl, -mn0));
            const float p1 = fast_exp2(fmaf(s[n][1], sl, -mn0));
            const float p2 = fast_exp2(fmaf(s[n][2], sl, -mn1));
            const float p3 = fast_exp2(fmaf(s[n][3], sl, -mn1));
            ps0 += p0 + p1;
            ps1 += p2 + p3;
            pf[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p0, p1);
            pf[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p2, p3);
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            oacc[n][0] *= al0;
            oacc[n][1] *= al0;
            oacc[n][2] *= al1;
            oacc[n][3] *= al1;
        }
        // O += P V ; P as A (16 x 64 keys), V stored [key][d]
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint32_t a[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t b[4];
                ldb_kn<CH>(sV, kk * 16, 2 * dp, b);
                mma_bf16(oacc[2 * dp], a, b[0], b[1]);
                mma_bf16(oacc[2 * dp + 1], a, b[2], b[3]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    const int g = lane >> 2, t = lane & 3;
    const int64_t row0 = bh * N + static_cast<int64_t>(i) * kBlk + warp * 16 + g;
    __nv_bfloat16 *o0 = o + row0 * D, *o1 = o + (row0 + 8) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        *reinterpret_cast<uint32_t *>(o0 + n * 8 + 2 * t) = pack_bf16(oacc[n][0] * inv0, oacc[n][1] * inv0);
        *reinterpret_cast<uint32_t *>(o1 + n * 8 + 2 * t) = pack_bf16(oacc[n][2] * inv1, oacc[n][3] * inv1);
    }
    if (lse != nullptr && t == 0) {
        lse[row0] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
        lse[row0 + 8] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
    }
}

// ---------------------------------------------------------------------------
// backward: D_n = dO_n . O_n  (16 threads per row)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16 *__restrict__ o,
                                                      const __nv_bfloat16 *__restrict__ dout,
                                                      float *__restrict__ dl, int64_t rows) {
    constexpr int TPR = 16;              // threads per row
    constexpr int EPT = D / TPR;         // elements per thread (8 or 4)
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / TPR;
    const int sub = threadIdx.x % TPR;
    float acc = 0.f;
    if (row < rows) {
        const __nv_bfloat16 *a = o + row * D + sub * EPT;
        const __nv_bfloat16 *b = dout + row * D + sub * EPT;
#pragma unroll
        for (int e = 0; e < EPT; e += 2) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(a + e));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(b + e));
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
    }
#pragma unroll
    for (int off = 1; off < TPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (row < rows && sub == 0) dl[row] = acc;
}

// ---------------------------------------------------------------------------
// backward: dK, dV for key block j over its column list
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) bwd_dkdv_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
    const float *__restrict__ lse, const float *__restrict__ dl,
    const uint16_t *__restrict__ col_idx, const int32_t *__restrict__ col_cnt,
    __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv, int nb, float scale) {
    constexpr int CH = D / 8;
    constexpr int TILE = kBlk * D * 2;
    constexpr int KT = D / 16;
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t sK = smem_addr(smem), sV = sK + TILE;
    const uint32_t sQ0 = sK + 2 * TILE, sO0 = sK + 4 * TILE;  // Q: [2], dO: [2]
    float *sL = reinterpret_cast<float *>(smem + 6 * TILE);   // [2][64] lse*log2e
    float *sD = sL + 2 * kBlk;                                // [2][64] D

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t bh = blockIdx.x / nb;
    const int j = blockIdx.x % nb;
    const int64_t N = static_cast<int64_t>(nb) * kBlk;
    const int cnt = col_cnt[bh * nb + j];
    const uint16_t *lst = col_idx + (bh * nb + j) * static_cast<int64_t>(nb);
    const __nv_bfloat16 *qh = q + bh * N * D, *doh = dout + bh * N * D;
    const float sl = scale * kLog2e;

    float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dka[n][e] = dva[n][e] = 0.f;

    load_tile<D>(sK, k + (bh * N + static_cast<int64_t>(j) * kBlk) * D, 128);
    load_tile<D>(sV, v + (bh * N + static_cast<int64_t>(j) * kBlk) * D, 128);
    auto stage = [&](int e, int buf) {
        const int i = lst[e];
        load_tile<D>(sQ0 + buf * TILE, qh + static_cast<int64_t>(i) * kBlk * D, 128);
        load_tile<D>(sO0 + buf * TILE, doh + static_cast<int64_t>(i) * kBlk * D, 128);
        if (threadIdx.x < kBlk) {
            const int64_t n = bh * N + static_cast<int64_t>(i) * kBlk + threadIdx.x;
            sL[buf * kBlk + threadIdx.x] = lse[n] * kLog2e;
            sD[buf * kBlk + threadIdx.x] = dl[n];
        }
    };
    if (cnt > 0) stage(0, 0);
    cp_async_commit();

    for (int e = 0; e < cnt; ++e) {
        const int buf = e & 1;
        if (e + 1 < cnt) {
            stage(e + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t sQ = sQ0 + buf * TILE, sO = sO0 + buf * TILE;
        const float *L = sL + buf * kBlk, *Dd = sD + buf * kBlk;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const int q0 = half * 32;
            // S^T (16 keys x 32 queries) and dP^T
            float s[4][4], dp[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int x = 0; x < 4; ++x) s[n][x] = dp[n][x] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
                uint32_t ka[4], va[4];
                lda<CH>(sK, warp * 16, kk, ka);
                lda<CH>(sV, warp * 16, kk, va);
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t b[4], c[4];
                    ldb_nk<CH>(sQ, q0 + np * 16, kk, b);
                    ldb_nk<CH>(sO, q0 + np * 16, kk, c);
                    mma_bf16(s[2 * np], ka, b[0], b[1]);
                    mma_bf16(s[2 * np + 1], ka, b[2], b[3]);
                    mma_bf16(dp[2 * np], va, c[0], c[1]);
                    mma_bf16(dp[2 * np + 1], va, c[2], c[3]);
                }
            }
            uint32_t pa[2][4], da[2][4];
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int qc = q0 + n * 8 + 2 * t;  // query columns qc, qc+1
                const float l0 = L[qc], l1 = L[qc + 1], d0 = Dd[qc], d1 = Dd[qc + 1];
                const float p00 = fast_exp2(fmaf(s[n][0], sl, -l0));
                const float p01 = fast_exp2(fmaf(s[n][1], sl, -l1));
                const float p10 = fast_exp2(fmaf(s[n][2], sl, -l0));
                const float p11 = fast_exp2(fmaf(s[n][3], sl, -l1));
                pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p00, p01);
                pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p10, p11);
                da[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p00 * (dp[n][0] - d0), p01 * (dp[n][1] - d1));
                da[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p10 * (dp[n][2] - d0), p11 * (dp[n][3] - d1));
            }
            // dV += P^T dO ; dK += dS^T Q  (k-dim = the 32 queries)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int dpi = 0; dpi < D / 16; ++dpi) {
                    uint32_t b[4], c[4];
                    ldb_kn<CH>(sO, q0 + kk * 16, 2 * dpi, b);
                    ldb_kn<CH>(sQ, q0 + kk * 16, 2 * dpi, c);
                    mma_bf16(dva[2 * dpi], pa[kk], b[0], b[1]);
                    mma_bf16(dva[2 * dpi + 1], pa[kk], b[2], b[3]);
                    mma_bf16(dka[2 * dpi], da[kk], c[0], c[1]);
                    mma_bf16(dka[2 * dpi + 1], da[kk], c[2], c[3]);
                }
            }
        }
        __syncthreads();
    }
    const int64_t row0 = bh * N + static_cast<int64_t>(j) * kBlk + warp * 16 + g;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        const int c = n * 8 + 2 * t;
        *reinterpret_cast<uint32_t *>(dk + row0 * D + c) = pack_bf16(dka[n][0] * scale, dka[n][1] * scale);
        *reinterpret_cast<uint32_t *>(dk + (row0 + 8) * D + c) = pack_bf16(dka[n][2] * scale, dka[n][3] * scale);
        *reinterpret_cast<uint32_t *>(dv + row0 * D + c) = pack_bf16(dva[n][0], dva[n][1]);
        *reinterpret_cast<uint32_t *>(dv + (row0 + 8) * D + c) = pack_bf16(dva[n][2], dva[n][3]);
    }
}

// ---------------------------------------------------------------------------
// backward: dQ for query block i over its row list
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) bwd_dq_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
    const float *__restrict__ lse, const float *__restrict__ dl,
    const uint16_t *__restrict__ row_idx, const int32_t *__restrict__ row_cnt,
    __nv_bfloat16 *__restrict__ dq, int nb, float scale) {
    constexpr int CH = D / 8;
    constexpr int TILE = kBlk * D * 2;
    constexpr int KT = D / 16;
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t sQ = smem_addr(smem), sO = sQ + TILE;
    const uint32_t sK0 = sQ + 2 * TILE, sV0 = sQ + 4 * TILE;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t bh = blockIdx.x / nb;
    const int i = blockIdx.x % nb;
    const int64_t N = static_cast<int64_t>(nb) * kBlk;
    const int cnt = row_cnt[bh * nb + i];
    const uint16_t *lst = row_idx + (bh * nb + i) * static_cast<int64_t>(nb);
    const __nv_bfloat16 *kh = k + bh * N * D, *vh = v + bh * N * D;
    const float sl = scale * kLog2e;
    const int64_t row0 = bh * N + static_cast<int64_t>(i) * kBlk + warp * 16 + g;
    const float L0 = lse[row0] * kLog2e, L1 = lse[row0 + 8] * kLog2e;
    const float D0 = dl[row0], D1 = dl[row0 + 8];

    float dqa[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) dqa[n][0] = dqa[n][1] = dqa[n][2] = dqa[n][3] = 0.f;

    load_tile<D>(sQ, q + (bh * N + static_cast<int64_t>(i) * kBlk) * D, 128);
    load_tile<D>(sO, dout + (bh * N + static_cast<int64_t>(i) * kBlk) * D, 128);
    if (cnt > 0) {
        const int j = lst[0];
        load_tile<D>(sK0, kh + static_cast<int64_t>(j) * kBlk * D, 128);
        load_tile<D>(sV0, vh + static_cast<int64_t>(j) * kBlk * D, 128);
    }
    cp_async_commit();
    for (int e = 0; e < cnt; ++e) {
        const int buf = e & 1;
        if (e + 1 < cnt) {
            const int j = lst[e + 1];
            load_tile<D>(sK0 + (buf ^ 1) * TILE, kh + static_cast<int64_t>(j) * kBlk * D, 128);
            load_tile<D>(sV0 + (buf ^ 1) * TILE, vh + static_cast<int64_t>(j) * kBlk * D, 128);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t sK = sK0 + buf * TILE, sV = sV0 + buf * TILE;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const int k0 = half * 32;
            float s[4][4], dp[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int x = 0; x < 4; ++x) s[n][x] = dp[n][x] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
                uint32_t qa[4], oa[4];
                lda<CH>(sQ, warp * 16, kk, qa);
                lda<CH>(sO, warp * 16, kk, oa);
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t b[4], c[4];
                    ldb_nk<CH>(sK, k0 + np * 16, kk, b);
                    ldb_nk<CH>(sV, k0 + np * 16, kk, c);
                    mma_bf16(s[2 * np], qa, b[0], b[1]);
                    mma_bf16(s[2 * np + 1], qa, b[2], b[3]);
                    mma_bf16(dp[2 * np], oa, c[0], c[1]);
                    mma_bf16(dp[2 * np + 1], oa, c[2], c[3]);
                }
            }
            uint32_t da[2][4];
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const float p0 = fast_exp2(fmaf(s[n][0], sl, -L0));
                const float p1 = fast_exp2(fmaf(s[n][1], sl, -L0));
                const float p2 = fast_exp2(fmaf(s[n][2], sl, -L1));
                const float p3 = fast_exp2(fmaf(s[n][3], sl, -L1));
                da[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p0 * (dp[n][0] - D0), p1 * (dp[n][1] - D0));
                da[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p2 * (dp[n][2] - D1), p3 * (dp[n][3] - D1));
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int dpi = 0; dpi < D / 16; ++dpi) {
                    uint32_t b[4];
                    ldb_kn<CH>(sK, k0 + kk * 16, 2 * dpi, b);
                    mma_bf16(dqa[2 * dpi], da[kk], b[0], b[1]);
                    mma_bf16(dqa[2 * dpi + 1], da[kk], b[2], b[3]);
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        const int c = n * 8 + 2 * t;
        *reinterpret_cast<uint32_t *>(dq + row0 * D + c) = pack_bf16(dqa[n][0] * scale, dqa[n][1] * scale);
        *reinterpret_cast<uint32_t *>(dq + (row0 + 8) * D + c) = pack_bf16(dqa[n][2] * scale, dqa[n][3] * scale);
    }
}

}  // namespace mma
}  // namespace nabla

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <int D>
static cudaError_t launch_fwd_mma(int64_t BH, int nb, float scale, const void *q, const void *k,
                                  const void *v, const uint16_t *row_idx, const int32_t *row_cnt,
                                  void *o, float *lse, cudaStream_t stream) {
    const int smem = 5 * nabla::kBlk * D * 2;
    cudaError_t err = cudaFuncSetAttribute(nabla::mma::fwd_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    nabla::mma::fwd_kernel<D><<<static_cast<unsigned>(BH * nb), 128, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), row_idx, row_cnt, static_cast<__nv_bfloat16 *>(o),
        lse, nb, scale);
    return cudaGetLastError();
}

cudaError_t nabla_launch_attn_fwd_mma(int64_t BH, int nb, int D, float scale, const void *q,
                                      const void *k, const void *v, const uint16_t *row_idx,
                                      const int32_t *row_cnt, void *o, float *lse,
                                      cudaStream_t stream) {
    return D == 128 ? launch_fwd_mma<128>(BH, nb, scale, q, k, v, row_idx, row_cnt, o, lse, stream)
                    : launch_fwd_mma<64>(BH, nb, scale, q, k, v, row_idx, row_cnt, o, lse, stream);
}

template <int D>
static cudaError_t launch_bwd_mma(int64_t BH, int nb, float scale, const void *q, const void *k,
                                  const void *v, const void *o, const void *dout, const float *lse,
                                  const uint16_t *row_idx, const int32_t *row_cnt,
                                  const uint16_t *col_idx, const int32_t *col_cnt, void *dq,
                                  void *dk, void *dv, float *dl, cudaStream_t stream) {
    using namespace nabla;
    const int64_t rows = BH * nb * static_cast<int64_t>(kBlk);
    mma::bwd_pre_kernel<D><<<static_cast<unsigned>((rows * 16 + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), dl, rows);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int smem_kv = 6 * kBlk * D * 2 + 4 * kBlk * static_cast<int>(sizeof(float));
    err = cudaFuncSetAttribute(mma::bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem_kv);
    if (err != cudaSuccess) return err;
    mma::bwd_dkdv_kernel<D><<<static_cast<unsigned>(BH * nb), 128, smem_kv, stream>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(dout), lse, dl,
        col_idx, col_cnt, static_cast<__nv_bfloat16 *>(dk), static_cast<__nv_bfloat16 *>(dv), nb,
        scale);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int smem_q = 6 * kBlk * D * 2;
    err = cudaFuncSetAttribute(mma::bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem_q);
    if (err != cudaSuccess) return err;
    mma::bwd_dq_kernel<D><<<static_cast<unsigned>(BH * nb), 128, smem_q, stream>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(dout), lse, dl,
        row_idx, row_cnt, static_cast<__nv_bfloat16 *>(dq), nb, scale);
    return cudaGetLastError();
}

cudaError_t nabla_launch_attn_bwd_mma(int64_t BH, int nb, int D, float scale, const void *q,
                                      const void *k, const void *v, const void *o,
                                      const void *dout, const float *lse, const uint16_t *row_idx,
                                      const int32_t *row_cnt, const uint16_t *col_idx,
                                      const int32_t *col_cnt, void *dq, void *dk, void *dv,
                                      float *dl, cudaStream_t stream) {
    return D == 128 ? launch_bwd_mma<128>(BH, nb, scale, q, k, v, o, dout, lse, row_idx, row_cnt,
                                          col_idx, col_cnt, dq, dk, dv, dl, stream)
                    : launch_bwd_mma<64>(BH, nb, scale, q, k, v, o, dout, lse, row_idx, row_cnt,
                                         col_idx, col_cnt, dq, dk, dv, dl, stream);
}
