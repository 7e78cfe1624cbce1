// Shared device helpers of the MATE token-mix library: scan-order and window
// index arithmetic, element loads/stores, block scans.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mate.h"

namespace mate {

// ---------------------------------------------------------------------------
// Rotary Major Scan (paper review, MA-Branch item 2): scan position n of a
// T x H x W grid -> grid offset (t*H + h)*W + w. Each order gives the three
// axes a priority; the first-priority axis varies fastest along the scan.
//   SR (W, H, T)   SC (H, W, T)   TR (T, W, H)   TC (T, H, W)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int rms_grid_offset(int n, int T, int H, int W, int mode)
{
    switch (mode) {
    case MATE_SCAN_SR:
        return n;
    case MATE_SCAN_SC: {
        const int hw = H * W;
        const int t = n / hw, r = n - t * hw;
        const int w = r / H, h = r - w * H;
        return t * hw + h * W + w;
    }
    case MATE_SCAN_TR: {
        const int s = n / T, t = n - s * T;
        const int h = s / W, w = s - h * W;
        return (t * H + h) * W + w;
    }
    case MATE_SCAN_ZZ: {  // 3D boustrophedon (mate.h)
        const int hw = H * W;
        const int t = n / hw, r = n - t * hw;
        const int i = r / W, j = r - i * W;
        const int h = (t & 1) ? H - 1 - i : i;
        const int w = ((t * H + i) & 1) ? W - 1 - j : j;
        return (t * H + h) * W + w;
    }
    default: {  // MATE_SCAN_TC
        const int s = n / T, t = n - s * T;
        const int w = s / H, h = s - w * H;
        return (t * H + h) * W + w;
    }
    }
}

// ---------------------------------------------------------------------------
// TESA windows (paper review, TE-Branch): along an axis of window size S and
// shift s, boundaries sit at coordinates congruent to s modulo S. Window k
// covers [k*S - off, (k+1)*S - off) clipped to the axis, off = (S - s) % S.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int win_offset(int S, int s) { return (S - s) % S; }
__host__ __device__ __forceinline__ int win_index(int c, int S, int off) { return (c + off) / S; }
__host__ __device__ __forceinline__ int win_count(int L, int S, int off) { return (L + off + S - 1) / S; }
__host__ __device__ __forceinline__ void win_range(int k, int L, int S, int off, int &lo, int &hi)
{
    lo = k * S - off;
    hi = lo + S;
    if (lo < 0) lo = 0;
    if (hi > L) hi = L;
}

// ---------------------------------------------------------------------------
// element access: fp32 compute on fp32 or bf16 storage
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float ld(const T *p);
template <> __device__ __forceinline__ float ld<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st(T *p, float v);
template <> __device__ __forceinline__ void st<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16 *p, float v)
{
    *p = __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------------------
// inclusive prefix sum over the first `n` entries of a shared array, for a
// block of any size (n <= blockDim.x * 32). All threads must call it.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_inclusive_scan(float v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sequential-in-warp-order inclusive scan of buf[0..n) in place, n <= 1024,
// using the first warp only (others wait at the trailing barrier).
__device__ __forceinline__ void block_inclusive_scan(float *buf, int n)
{
    __syncthreads();
    if (threadIdx.x < 32) {
        float carry = 0.f;
        for (int base = 0; base < n; base += 32) {
            const int i = base + threadIdx.x;
            float v = i < n ? buf[i] : 0.f;
            v = warp_inclusive_scan(v) + carry;
            if (i < n) buf[i] = v;
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();
}

}  // namespace mate
