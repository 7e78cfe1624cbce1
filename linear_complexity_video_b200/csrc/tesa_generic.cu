// TEmporal Swin Attention, CUDA-core path for fp32 storage, any supported head
// size and window (bf16 storage runs on the tensor-core kernel of tesa_tc.cu).
//
// Method (paper review "LinGen ...", section 三, TE-Branch): each token
// attends only to the tokens of its Tw x Sw x Sw window; the window grid is
// shifted on alternate layers. Along each axis the window boundaries sit at
// coordinates congruent to the shift modulo the window size, so shifted
// grids have partial windows at both ends.
//
// One CTA per (window, head, batch element). K and V of the window are
// staged in shared memory; one warp per query row runs an online softmax
// over the window's keys, lanes splitting the head dimension.
#include "common.cuh"
#include "kernels.h"

namespace mate {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void window_box(const TesaArgs &a, int wid, int &t0, int &lt, int &h0, int &lh, int &w0,
                                           int &lw)
{
    const int kw = wid % a.nww;
    const int r = wid / a.nww;
    const int kh = r % a.nwh;
    const int kt = r / a.nwh;
    int t1, h1, w1;
    win_range(kt, a.T, a.Tw, a.offt, t0, t1);
    win_range(kh, a.H, a.Sw, a.offh, h0, h1);
    win_range(kw, a.W, a.Sw, a.offw, w0, w1);
    lt = t1 - t0;
    lh = h1 - h0;
    lw = w1 - w0;
}

template <typename T, int DH>
__global__ void __launch_bounds__(kThreads) tesa_generic_kernel(TesaArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int EPL = (DH + 31) / 32;  // head-dim elements per lane
    const int wid = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    int t0, lt, h0, lh, w0, lw;
    window_box(a, wid, t0, lt, h0, lh, w0, lw);
    const int m = lt * lh * lw;
    T *ks = reinterpret_cast<T *>(smem_raw);
    T *vs = ks + (size_t)m * DH;
    int *goff = reinterpret_cast<int *>(vs + (size_t)m * DH);
    const T *q = static_cast<const T *>(a.q);
    const T *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v);
    T *out = static_cast<T *>(a.out);

    for (int i = threadIdx.x; i < m; i += blockDim.x) {
        const int it = i / (lh * lw), r = i - it * (lh * lw), ih = r / lw, iw = r - ih * lw;
        goff[i] = ((t0 + it) * a.H + h0 + ih) * a.W + w0 + iw;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < m * DH; idx += blockDim.x) {
        const int i = idx / DH, e = idx - i * DH;
        const size_t off = (((size_t)b * a.N + goff[i]) * a.nh + h) * DH + e;
        ks[idx] = k[off];
        vs[idx] = v[off];
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const float scale = rsqrtf((float)DH);
    for (int i = warp; i < m; i += nwarps) {
        const size_t row = (((size_t)b * a.N + goff[i]) * a.nh + h) * DH;
        float qv[EPL], acc[EPL];
#pragma unroll
        for (int u = 0; u < EPL; ++u) {
            const int e = lane + 32 * u;
            qv[u] = e < DH ? ld(q + row + e) * scale : 0.f;
            acc[u] = 0.f;
        }
        float mx = -INFINITY, den = 0.f;
        for (int j = 0; j < m; ++j) {
            float part = 0.f;
#pragma unroll
            for (int u = 0; u < EPL; ++u) {
                const int e = lane + 32 * u;
                if (e < DH) part += qv[u] * ld(ks + (size_t)j * DH + e);
            }
            const float sc = warp_sum(part);
            const float mnew = fmaxf(mx, sc);
            const float corr = expf(mx - mnew);
            const float p = expf(sc - mnew);
            den = den * corr + p;
#pragma unroll
            for (int u = 0; u < EPL; ++u) {
                const int e = lane + 32 * u;
                const float vv = e < DH ? ld(vs + (size_t)j * DH + e) : 0.f;
                acc[u] = acc[u] * corr + p * vv;
            }
            mx = mnew;
        }
        const float inv = 1.f / den;
#pragma unroll
        for (int u = 0; u < EPL; ++u) {
            const int e = lane + 32 * u;
            if (e < DH) st(out + row + e, acc[u] * inv);
        }
    }
}

template <typename T, int DH>
cudaError_t run(const TesaArgs &a, cudaStream_t s)
{
    const int maxm = a.Tw * a.Sw * a.Sw;
    const size_t smem = (size_t)maxm * DH * sizeof(T) * 2 + (size_t)maxm * sizeof(int);
    cudaError_t e =
        cudaFuncSetAttribute(tesa_generic_kernel<T, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nwin = a.nwt * a.nwh * a.nww;
    Phase ph(MATE_PHASE_TESA, s);
    tesa_generic_kernel<T, DH><<<dim3(nwin, a.nh, a.batch), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const TesaArgs &a, cudaStream_t s)
{
    switch (a.d) {
    case 16: return run<T, 16>(a, s);
    case 32: return run<T, 32>(a, s);
    case 64: return run<T, 64>(a, s);
    case 128: return run<T, 128>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

__global__ void tesa_map_kernel(TesaArgs a, int32_t *out)
{
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= a.N) return;
    const int hw = a.H * a.W;
    const int t = g / hw, r = g - t * hw, hh = r / a.W, w = r - hh * a.W;
    const int kt = win_index(t, a.Tw, a.offt), kh = win_index(hh, a.Sw, a.offh), kw = win_index(w, a.Sw, a.offw);
    out[g] = (kt * a.nwh + kh) * a.nww + kw;
}

__global__ void rms_map_kernel(int T, int H, int W, int mode, int flip, int32_t *out)
{
    const int N = T * H * W;
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    out[n] = rms_grid_offset(flip ? N - 1 - n : n, T, H, W, mode);
}

}  // namespace

cudaError_t launch_tesa_generic(const TesaArgs &a, cudaStream_t s)
{
    // fp32 storage only: bf16 calls run on the tensor-core kernel or are refused
    return a.bf16 ? cudaErrorInvalidValue : dispatch<float>(a, s);
}

cudaError_t launch_tesa_map(const TesaArgs &a, int32_t *out, cudaStream_t s)
{
    tesa_map_kernel<<<(a.N + 255) / 256, 256, 0, s>>>(a, out);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_rms_map(int T, int H, int W, int mode, int flip, int32_t *out, cudaStream_t s)
{
    const int N = T * H * W;
    rms_map_kernel<<<(N + 255) / 256, 256, 0, s>>>(T, H, W, mode, flip, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace mate
