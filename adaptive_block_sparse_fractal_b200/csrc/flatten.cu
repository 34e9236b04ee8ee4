// Fractal flattening ("NABLA: Neighborhood Adaptive Block-Level Attention",
// section 手法: NABLA, "トークン再順序付け (Fractal Flattening)").
//
// Token (t, y, x) of a T x H x W grid moves to
//   n = ((t*Hp + y/P)*Wp + x/P)*P*P + (y%P)*P + x%P,   Hp = H/P, Wp = W/P.
// The P tokens of one patch row (t, y, x0..x0+P-1) are contiguous on both
// sides, so the copy is a set of runs of P*inner_bytes bytes (2 KiB for P=8,
// bf16, D=128).  One warp moves one run with 16-byte vector loads/stores; the
// index arithmetic is paid once per run.  HBM-bound: 2 * bytes moved.
#include "common.cuh"

namespace nabla {

__global__ void __launch_bounds__(256) flatten_kernel(const uint8_t *__restrict__ in,
                                                      uint8_t *__restrict__ out, int64_t runs,
                                                      int H, int W, int P, int64_t inner_bytes,
                                                      int inverse) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int Hp = H / P, Wp = W / P;
    const int64_t HW = static_cast<int64_t>(H) * W;
    const int64_t run_bytes = P * inner_bytes;
    const int64_t chunks = run_bytes >> 4;
    // A run is (outer-frame f = o*T + t, patch row y, patch column pw).
    for (int64_t r = warp; r < runs; r += nwarps) {
        const int pw = static_cast<int>(r % Wp);
        const int64_t ry = r / Wp;
        const int y = static_cast<int>(ry % H);
        const int64_t f = ry / H;  // o*T + t
        const int64_t base = f * HW;
        const int64_t n_grid = base + static_cast<int64_t>(y) * W + static_cast<int64_t>(pw) * P;
        const int64_t n_flat = base + ((static_cast<int64_t>(y / P) * Wp + pw) * P + (y % P)) * P;
        const int64_t src_tok = inverse ? n_flat : n_grid;
        const int64_t dst_tok = inverse ? n_grid : n_flat;
        const int4 *src = reinterpret_cast<const int4 *>(in + src_tok * inner_bytes);
        int4 *dst = reinterpret_cast<int4 *>(out + dst_tok * inner_bytes);
        int64_t c = lane;
        for (; c + 96 < chunks; c += 128) {
            int4 a = __ldg(src + c), b = __ldg(src + c + 32), d = __ldg(src + c + 64),
                 e = __ldg(src + c + 96);
            __stcs(dst + c, a);
            __stcs(dst + c + 32, b);
            __stcs(dst + c + 64, d);
            __stcs(dst + c + 96, e);
        }
        for (; c < chunks; c += 32) __stcs(dst + c, __ldg(src + c));
    }
    (void)Hp;
}

}  // namespace nabla

// Launcher used by the C ABI layer.
cudaError_t nabla_launch_flatten(const void *in, void *out, int64_t outer, int T, int H, int W,
                                 int P, int64_t inner_bytes, int inverse, cudaStream_t stream) {
    const int64_t runs = outer * T * static_cast<int64_t>(H) * (W / P);
    if (runs == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps_per_block = 8;
    int64_t blocks = (runs + warps_per_block - 1) / warps_per_block;
    const int64_t cap = static_cast<int64_t>(sms) * 16;  // 16 resident blocks of 256 per SM
    if (blocks > cap) blocks = cap;
    nabla::flatten_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint8_t *>(in), static_cast<uint8_t *>(out), runs, H, W, P, inner_bytes,
        inverse);
    return cudaGetLastError();
}
