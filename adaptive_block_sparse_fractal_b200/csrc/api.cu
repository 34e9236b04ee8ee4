// C ABI of libnabla.so (declared in include/nabla.h): argument checks,
// workspace layout, status word, kernel dispatch.  Every host-detectable
// error is returned before anything is enqueued.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/nabla.h"
#include "common.cuh"

// launchers (mask.cu, flatten.cu, attn_*.cu)
cudaError_t nabla_launch_flatten(const void *in, void *out, int64_t outer, int T, int H, int W,
                                 int P, int64_t inner_bytes, int inverse, cudaStream_t stream);
cudaError_t nabla_launch_build_mask(int64_t BH, int nb, int D, int T, int Hp, int Wp, float p,
                                    float scale, int wt, int wh, int ww, unsigned flags,
                                    const void *q, const void *k, float *qbar, float *kbar_t,
                                    uint32_t *bits, uint16_t *row_idx, int32_t *row_cnt,
                                    uint16_t *col_idx, int32_t *col_cnt, float *scores,
                                    cudaStream_t stream, const void *q_grid, const void *k_grid,
                                    int *ctr, int *status);
cudaError_t nabla_launch_build_mask_dr(int64_t BH, int nb, int D, int T, int Hp, int Wp, int mode,
                                       double gamma, double lambda, float tau, float scale, int wt,
                                       int wh, int ww, unsigned flags, const void *q,
                                       const void *k, float *qbar, float *kbar_t, uint32_t *bits,
                                       uint16_t *row_idx, int32_t *row_cnt, uint16_t *col_idx,
                                       int32_t *col_cnt, float *scores, cudaStream_t stream);
cudaError_t nabla_launch_attn_fwd_sm100(int64_t BH, int nb, int D, int Hp, int Wp, int T,
                                        float scale, const void *q, const void *k, const void *v,
                                        const uint32_t *bits, void *o, float *lse, int *status,
                                        int force_timeout, cudaStream_t stream);
cudaError_t nabla_launch_attn_bwd_sm100(int64_t BH, int nb, int D, int Hp, int Wp, int T,
                                        float scale, const void *q, const void *k, const void *v,
                                        const void *o, const void *dout, const float *lse,
                                        const uint16_t *row_idx, const int32_t *row_cnt,
                                        const uint16_t *col_idx, const int32_t *col_cnt,
                                        void *dq, void *dk, void *dv, float *dl, float *l2,
                                        int *status, int force_timeout, cudaStream_t stream);

namespace {

constexpr size_t kStatusBytes = 256;
constexpr int kMaxNb = 2048;

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Scratch of the mask build: pooled Q [BH, nb, D] then pooled K transposed
// [BH, D, nbp] (nbp = nb rounded up to a multiple of 4).  In a workspace they
// follow the status region and the task counters of the persistent front end
// (1 + BH ints).
struct MaskScratch {
    size_t qbar_bytes, kbar_bytes;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Dims {
    int64_t BH, N;
    int nb, D, Hp, Wp;
};

int check_shape(const nabla_shape *s, Dims *d) {
    if (s == nullptr) return NABLA_ERR_NULL;
    if (s->B < 1 || s->heads < 1 || s->T < 1 || s->H < 1 || s->W < 1) return NABLA_ERR_SHAPE;
    if (s->P != 8 || s->H % s->P != 0 || s->W % s->P != 0) return NABLA_ERR_SHAPE;
    if (s->D != 64 && s->D != 128) return NABLA_ERR_SHAPE;
    const int64_t nb = static_cast<int64_t>(s->T) * (s->H / s->P) * (s->W / s->P);
    if (nb < 1 || nb > kMaxNb) return NABLA_ERR_SHAPE;
    d->BH = static_cast<int64_t>(s->B) * s->heads;
    d->nb = static_cast<int>(nb);
    d->N = nb * nabla::kBlk;
    d->D = s->D;
    d->Hp = s->H / s->P;
    d->Wp = s->W / s->P;
    return NABLA_OK;
}

int check_params(const nabla_params *p, bool need_window) {
    if (p == nullptr) return NABLA_ERR_NULL;
    if (!(p->p >= 0.f && p->p <= 1.f)) return NABLA_ERR_PARAM;  // also rejects NaN
    if (!(p->scale > 0.f) || !std::isfinite(p->scale)) return NABLA_ERR_PARAM;
    if ((p->flags & ~(NABLA_NO_STA | NABLA_FULL_STA | NABLA_EMIT_COLS | NABLA_DEBUG_SCORES |
                      NABLA_DEBUG_TIMEOUT)) != 0)
        return NABLA_ERR_PARAM;
    if ((p->flags & NABLA_NO_STA) && (p->flags & NABLA_FULL_STA)) return NABLA_ERR_PARAM;
    if (need_window && !(p->flags & (NABLA_NO_STA | NABLA_FULL_STA))) {
        for (int w : {p->sta_t, p->sta_h, p->sta_w})
            if (w < 1 || (w & 1) == 0) return NABLA_ERR_PARAM;
    }
    return NABLA_OK;
}

MaskScratch mask_scratch(const Dims &d) {
    const size_t nbp = (static_cast<size_t>(d.nb) + 3) & ~static_cast<size_t>(3);
    return {round256(sizeof(float) * d.BH * d.nb * d.D), round256(sizeof(float) * d.BH * d.D * nbp)};
}

size_t mask_scratch_bytes(const Dims &d) {
    const MaskScratch m = mask_scratch(d);
    return m.qbar_bytes + m.kbar_bytes;
}

size_t counter_bytes(const Dims &d) { return round256(sizeof(int) * (1 + d.BH)); }

size_t ws_bytes(const Dims &d, int op) {
    switch (op) {
        case NABLA_OP_BUILD_MASK:
            return kStatusBytes + counter_bytes(d) + mask_scratch_bytes(d);
        case NABLA_OP_ATTN_FWD:
            return kStatusBytes;
        case NABLA_OP_ATTN_BWD:  // D_n and lse_n * log2(e)
            return kStatusBytes + 2 * round256(sizeof(float) * d.BH * d.N);
        default:
            return 0;
    }
}

int check_ws(const Dims &d, int op, void *ws, size_t bytes) {
    if (ws == nullptr || bytes < ws_bytes(d, op)) return NABLA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return NABLA_ERR_ALIGN;
    return NABLA_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? NABLA_OK : NABLA_ERR_CUDA; }

int clear_status(void *ws, cudaStream_t s) {
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int), s));
}

bool overlap(const void *a, const void *b, size_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

// Pointer checks shared by the three mask-building calls.
int check_mask_ptrs(const nabla_params *params, const nabla_mask *mask) {
    if (mask == nullptr || mask->bits == nullptr || mask->row_idx == nullptr ||
        mask->row_cnt == nullptr)
        return NABLA_ERR_NULL;
    if ((params->flags & NABLA_EMIT_COLS) && (mask->col_idx == nullptr || mask->col_cnt == nullptr))
        return NABLA_ERR_NULL;
    if ((params->flags & NABLA_DEBUG_SCORES) && mask->scores == nullptr) return NABLA_ERR_NULL;
    return NABLA_OK;
}

float *debug_scores(const nabla_params *params, const nabla_mask *mask) {
    return (params->flags & NABLA_DEBUG_SCORES) ? mask->scores : nullptr;
}

}  // namespace

extern "C" {

int nabla_flatten(const void *in, void *out, int64_t outer, int T, int H, int W, int P,
                  int64_t inner_bytes, int inverse, nabla_stream_t stream) {
    if (outer < 0 || T < 0 || H < 0 || W < 0 || P < 1 || inner_bytes < 0) return NABLA_ERR_SHAPE;
    if (H % P != 0 || W % P != 0) return NABLA_ERR_SHAPE;
    if (inner_bytes % 16 != 0) return NABLA_ERR_ALIGN;
    if (outer == 0 || T == 0 || H == 0 || W == 0 || inner_bytes == 0) return NABLA_OK;  // empty
    if (in == nullptr || out == nullptr) return NABLA_ERR_NULL;
    if (!aligned16(in) || !aligned16(out)) return NABLA_ERR_ALIGN;
    const size_t bytes = static_cast<size_t>(outer) * T * H * W * static_cast<size_t>(inner_bytes);
    if (overlap(in, out, bytes)) return NABLA_ERR_PARAM;
    return cuda_status(nabla_launch_flatten(in, out, outer, T, H, W, P, inner_bytes, inverse,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

size_t nabla_workspace_size(const nabla_shape *shape, int op) {
    Dims d;
    if (check_shape(shape, &d) != NABLA_OK) return 0;
    return ws_bytes(d, op);
}

size_t nabla_mask_bytes(const nabla_shape *shape, int part) {
    Dims d;
    if (check_shape(shape, &d) != NABLA_OK) return 0;
    const size_t rows = static_cast<size_t>(d.BH) * d.nb;
    switch (part) {
        case NABLA_MASK_BITS:
            return rows * ((d.nb + 31) / 32) * sizeof(uint32_t);
        case NABLA_MASK_ROW_IDX:
        case NABLA_MASK_COL_IDX:
            return rows * d.nb * sizeof(uint16_t);
        case NABLA_MASK_ROW_CNT:
        case NABLA_MASK_COL_CNT:
            return rows * sizeof(int32_t);
        case NABLA_MASK_SCORES:
            return rows * d.nb * sizeof(float);
        default:
            return 0;
    }
}

int nabla_build_mask(const nabla_shape *shape, const nabla_params *params, const nabla_bf16 *q,
                     const nabla_bf16 *k, const nabla_mask *mask, void *workspace,
                     size_t workspace_bytes, nabla_stream_t stream) {
    Dims d;
    int st = check_shape(shape, &d);
    if (st != NABLA_OK) return st;
    if ((st = check_params(params, true)) != NABLA_OK) return st;
    if (q == nullptr || k == nullptr) return NABLA_ERR_NULL;
    if ((st = check_mask_ptrs(params, mask)) != NABLA_OK) return st;
    const bool cols = (params->flags & NABLA_EMIT_COLS) != 0;
    if (!aligned16(q) || !aligned16(k)) return NABLA_ERR_ALIGN;
    if ((st = check_ws(d, NABLA_OP_BUILD_MASK, workspace, workspace_bytes)) != NABLA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != NABLA_OK) return st;
    int *ctr = reinterpret_cast<int *>(static_cast<unsigned char *>(workspace) + kStatusBytes);
    unsigned char *w = reinterpret_cast<unsigned char *>(ctr) + counter_bytes(d);
    float *qbar = reinterpret_cast<float *>(w);
    float *kbar_t = reinterpret_cast<float *>(w + mask_scratch(d).qbar_bytes);
    return cuda_status(nabla_launch_build_mask(
        d.BH, d.nb, d.D, shape->T, d.Hp, d.Wp, params->p, params->scale, params->sta_t,
        params->sta_h, params->sta_w, params->flags, q, k, qbar, kbar_t, mask->bits,
        mask->row_idx, mask->row_cnt, cols ? mask->col_idx : nullptr,
        cols ? mask->col_cnt : nullptr, debug_scores(params, mask), s, nullptr, nullptr, ctr,
        static_cast<int *>(workspace)));
}

int nabla_build_mask_grid(const nabla_shape *shape, const nabla_params *params,
                          const nabla_bf16 *q_grid, const nabla_bf16 *k_grid, nabla_bf16 *q,
                          nabla_bf16 *k, const nabla_mask *mask, void *workspace,
                          size_t workspace_bytes, nabla_stream_t stream) {
    Dims d;
    int st = check_shape(shape, &d);
    if (st != NABLA_OK) return st;
    if ((st = check_params(params, true)) != NABLA_OK) return st;
    if (q_grid == nullptr || k_grid == nullptr || q == nullptr || k == nullptr)
        return NABLA_ERR_NULL;
    if ((st = check_mask_ptrs(params, mask)) != NABLA_OK) return st;
    const bool cols = (params->flags & NABLA_EMIT_COLS) != 0;
    if (!aligned16(q_grid) || !aligned16(k_grid) || !aligned16(q) || !aligned16(k))
        return NABLA_ERR_ALIGN;
    // the flattened outputs must not overlap each other or either input
    const size_t bytes = sizeof(nabla_bf16) * static_cast<size_t>(d.BH) * d.N * d.D;
    if (overlap(q, k, bytes) || overlap(q, q_grid, bytes) || overlap(q, k_grid, bytes) ||
        overlap(k, q_grid, bytes) || overlap(k, k_grid, bytes))
        return NABLA_ERR_PARAM;
    if ((st = check_ws(d, NABLA_OP_BUILD_MASK, workspace, workspace_bytes)) != NABLA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != NABLA_OK) return st;
    int *ctr = reinterpret_cast<int *>(static_cast<unsigned char *>(workspace) + kStatusBytes);
    unsigned char *w = reinterpret_cast<unsigned char *>(ctr) + counter_bytes(d);
    float *qbar = reinterpret_cast<float *>(w);
    float *kbar_t = reinterpret_cast<float *>(w + mask_scratch(d).qbar_bytes);
    return cuda_status(nabla_launch_build_mask(
        d.BH, d.nb, d.D, shape->T, d.Hp, d.Wp, params->p, params->scale, params->sta_t,
        params->sta_h, params->sta_w, params->flags, q, k, qbar, kbar_t, mask->bits,
        mask->row_idx, mask->row_cnt, cols ? mask->col_idx : nullptr,
        cols ? mask->col_cnt : nullptr, debug_scores(params, mask), s, q_grid, k_grid, ctr,
        static_cast<int *>(workspace)));
}

int nabla_build_mask_dr(const nabla_shape *shape, const nabla_dr_params *params,
                        const nabla_bf16 *q, const nabla_bf16 *k, const nabla_mask *mask,
                        void *workspace, size_t workspace_bytes, nabla_stream_t stream) {
    Dims d;
    int st = check_shape(shape, &d);
    if (st != NABLA_OK) return st;
    if (params == nullptr) return NABLA_ERR_NULL;
    const bool thr = params->mode == NABLA_DR_THRESHOLD;
    if (!thr && params->mode != NABLA_DR_STATIC_RATIO) return NABLA_ERR_PARAM;
    // the window, scale and flag rules of nabla_params (p is not used)
    const nabla_params common{1.0f, params->sta_t, params->sta_h, params->sta_w, params->scale,
                              params->flags};
    if ((st = check_params(&common, true)) != NABLA_OK) return st;
    if (params->flags & NABLA_DEBUG_TIMEOUT) return NABLA_ERR_PARAM;
    if (!thr && (params->flags & NABLA_DEBUG_SCORES)) return NABLA_ERR_PARAM;  // no scores
    if (!(params->gamma > 0.0 && params->gamma <= 1.0)) return NABLA_ERR_PARAM;
    if (!(params->lambda >= 0.0 && params->lambda <= 1.0)) return NABLA_ERR_PARAM;
    if (!(params->tau >= 0.0f)) return NABLA_ERR_PARAM;  // also rejects NaN; infinity keeps all
    if ((st = check_mask_ptrs(&common, mask)) != NABLA_OK) return st;
    if (thr) {
        if (q == nullptr || k == nullptr) return NABLA_ERR_NULL;
        if (!aligned16(q) || !aligned16(k)) return NABLA_ERR_ALIGN;
    }
    const int op = thr ? NABLA_OP_BUILD_MASK : NABLA_OP_ATTN_FWD;  // the latter: status only
    if ((st = check_ws(d, op, workspace, workspace_bytes)) != NABLA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != NABLA_OK) return st;
    unsigned char *w = static_cast<unsigned char *>(workspace) + kStatusBytes + counter_bytes(d);
    float *qbar = thr ? reinterpret_cast<float *>(w) : nullptr;
    float *kbar_t = thr ? reinterpret_cast<float *>(w + mask_scratch(d).qbar_bytes) : nullptr;
    const bool cols = (params->flags & NABLA_EMIT_COLS) != 0;
    return cuda_status(nabla_launch_build_mask_dr(
        d.BH, d.nb, d.D, shape->T, d.Hp, d.Wp, params->mode, params->gamma, params->lambda,
        params->tau, params->scale, params->sta_t, params->sta_h, params->sta_w, params->flags, q,
        k, qbar, kbar_t, mask->bits, mask->row_idx, mask->row_cnt, cols ? mask->col_idx : nullptr,
        cols ? mask->col_cnt : nullptr, debug_scores(&common, mask), s));
}

int nabla_attn_fwd(const nabla_shape *shape, const nabla_params *params, const nabla_bf16 *q,
                   const nabla_bf16 *k, const nabla_bf16 *v, const nabla_mask *mask,
                   nabla_bf16 *o, float *lse, void *workspace, size_t workspace_bytes,
                   nabla_stream_t stream) {
    Dims d;
    int st = check_shape(shape, &d);
    if (st != NABLA_OK) return st;
    if ((st = check_params(params, false)) != NABLA_OK) return st;
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || mask == nullptr ||
        mask->bits == nullptr || mask->row_idx == nullptr || mask->row_cnt == nullptr)
        return NABLA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return NABLA_ERR_ALIGN;
    if ((st = check_ws(d, NABLA_OP_ATTN_FWD, workspace, workspace_bytes)) != NABLA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != NABLA_OK) return st;
    return cuda_status(nabla_launch_attn_fwd_sm100(
        d.BH, d.nb, d.D, d.Hp, d.Wp, shape->T, params->scale, q, k, v, mask->bits, o, lse,
        static_cast<int *>(workspace), (params->flags & NABLA_DEBUG_TIMEOUT) ? 1 : 0, s));
}

int nabla_attn_bwd(const nabla_shape *shape, const nabla_params *params, const nabla_bf16 *q,
                   const nabla_bf16 *k, const nabla_bf16 *v, const nabla_bf16 *o,
                   const nabla_bf16 *dout, const float *lse, const nabla_mask *mask,
                   nabla_bf16 *dq, nabla_bf16 *dk, nabla_bf16 *dv, void *workspace,
                   size_t workspace_bytes, nabla_stream_t stream) {
    Dims d;
    int st = check_shape(shape, &d);
    if (st != NABLA_OK) return st;
    if ((st = check_params(params, false)) != NABLA_OK) return st;
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || dout == nullptr ||
        lse == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || mask == nullptr ||
        mask->row_idx == nullptr || mask->row_cnt == nullptr || mask->col_idx == nullptr ||
        mask->col_cnt == nullptr)
        return NABLA_ERR_NULL;
    for (const void *p : {static_cast<const void *>(q), static_cast<const void *>(k),
                          static_cast<const void *>(v), static_cast<const void *>(o),
                          static_cast<const void *>(dout), static_cast<const void *>(dq),
                          static_cast<const void *>(dk), static_cast<const void *>(dv)})
        if (!aligned16(p)) return NABLA_ERR_ALIGN;
    if ((st = check_ws(d, NABLA_OP_ATTN_BWD, workspace, workspace_bytes)) != NABLA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != NABLA_OK) return st;
    float *dl = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + kStatusBytes);
    float *l2 = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(dl) +
                                          round256(sizeof(float) * d.BH * d.N));
    return cuda_status(nabla_launch_attn_bwd_sm100(
        d.BH, d.nb, d.D, d.Hp, d.Wp, shape->T, params->scale, q, k, v, o, dout, lse,
        mask->row_idx, mask->row_cnt, mask->col_idx, mask->col_cnt, dq, dk, dv, dl, l2,
        static_cast<int *>(workspace), (params->flags & NABLA_DEBUG_TIMEOUT) ? 1 : 0, s));
}

int nabla_status(const void *workspace, nabla_stream_t stream) {
    if (workspace == nullptr) return NABLA_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return NABLA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return NABLA_ERR_CUDA;
    return word == nabla::kDevOk ? NABLA_OK : NABLA_ERR_TIMEOUT;
}

const char *nabla_strerror(int status) {
    switch (status) {
        case NABLA_OK: return "ok";
        case NABLA_ERR_SHAPE: return "unsupported or inconsistent shape";
        case NABLA_ERR_ALIGN: return "pointer or byte count not 16-byte aligned";
        case NABLA_ERR_PARAM: return "invalid parameter";
        case NABLA_ERR_WORKSPACE: return "workspace missing or too small";
        case NABLA_ERR_CUDA: return "CUDA call or kernel launch failed";
        case NABLA_ERR_TIMEOUT: return "device-side bounded wait expired";
        case NABLA_ERR_NULL: return "required pointer is NULL";
        default: return "unknown status";
    }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// nabla_build_mask_static: the mask build with its scratch (the pooled means)
// in an array compiled into this library instead of a caller workspace.  For
// callers that are handed only their input and output buffers and may not
// call cudaMalloc themselves.  The array is allocated once per GPU when the
// library's device code is loaded there and held until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_mask_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];  // device address of g_mask_scratch, per device
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.  The first call
// on a device looks it up (the host-side name is only a stand-in, never a
// device address) and caches it.
int static_scratch(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NABLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mask_scratch) != cudaSuccess || p == nullptr)
            return NABLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return NABLA_OK;
}

}  // namespace

extern "C" int nabla_build_mask_static(const nabla_shape *shape, const nabla_params *params,
                                       const nabla_bf16 *q, const nabla_bf16 *k,
                                       const nabla_mask *mask, nabla_stream_t stream) {
    Dims d;
    int st = check_shape(shape, &d);
    if (st != NABLA_OK) return st;
    if ((st = check_params(params, true)) != NABLA_OK) return st;
    if (q == nullptr || k == nullptr) return NABLA_ERR_NULL;
    if ((st = check_mask_ptrs(params, mask)) != NABLA_OK) return st;
    const bool cols = (params->flags & NABLA_EMIT_COLS) != 0;
    if (!aligned16(q) || !aligned16(k)) return NABLA_ERR_ALIGN;
    const MaskScratch ms = mask_scratch(d);
    if (ms.qbar_bytes + ms.kbar_bytes > kStaticScratchBytes) return NABLA_ERR_WORKSPACE;
    void *base = nullptr;
    if ((st = static_scratch(&base)) != NABLA_OK) return st;
    // Every byte of the scratch that this call reads is written earlier in the
    // same call (pool kernel), so nothing has to be cleared first.
    float *qbar = static_cast<float *>(base);
    float *kbar_t = reinterpret_cast<float *>(static_cast<unsigned char *>(base) + ms.qbar_bytes);
    return cuda_status(nabla_launch_build_mask(
        d.BH, d.nb, d.D, shape->T, d.Hp, d.Wp, params->p, params->scale, params->sta_t,
        params->sta_h, params->sta_w, params->flags, q, k, qbar, kbar_t, mask->bits,
        mask->row_idx, mask->row_cnt, cols ? mask->col_idx : nullptr,
        cols ? mask->col_cnt : nullptr, debug_scores(params, mask),
        reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, nullptr));
}
