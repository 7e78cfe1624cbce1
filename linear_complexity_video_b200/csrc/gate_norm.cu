// MA-branch output side: the bi-SSD output y gated by the front-end's z and
// RMS-normalised per group of channels (paper review "LinGen ...", section 三,
// MA-Branch item 1: the branch is a bidirectional Mamba2 block; the pages name
// the block and no more of it, so this is the standard Mamba2 gated norm, gate
// first):
//     v_k   = y_k SiLU(z_k)
//     out_k = v_k w_k / sqrt(mean_{k in group} v_k^2 + eps)
// Its output is the MA-branch's input to the MATE composition.
//
// HBM-bound (y and z read once, out written once: 6 bytes per channel in bf16).
// One CTA of 128 threads per token row: thread t holds the 16-byte vectors
// t, t + 128, ... of the row (eight channels each, all loads in flight at once),
// so that every load and store instruction of a warp covers 512 contiguous bytes.
// The sums of squares go per vector to shared memory, warp w reduces groups
// w, w + 4, ... there, and each thread scales its vectors by its groups' factors.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

#include <cuda_bf16.h>

namespace mate {

namespace {

constexpr int kGnThreads = 128;
constexpr int kGnMaxVec = 8;  // vectors per thread: rows of up to 8 x 8 x 128 = 8192 channels

// SiLU(v) = v / (1 + e^-v) with the fast exponential and divide (relative error
// far below the bf16 rounding of the result, for either sign of v)
__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.f + __expf(-v)); }

__global__ void __launch_bounds__(kGnThreads) gate_norm_kernel(GateNormArgs a)
{
    __shared__ float ss_vec[kGnMaxVec * kGnThreads];  // sum of squares of each vector of the row
    __shared__ float scale[kGnMaxVec * kGnThreads];   // 1 / rms of each group (at most one per vector)
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int nv = a.C / 8, gv = a.group / 8, ng = a.C / a.group;  // vectors per row, per group; groups
    const size_t row = (size_t)blockIdx.x * a.C;
    const uint4 *y = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.y) + row);
    const uint4 *z = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.z) + row);
    uint4 yv[kGnMaxVec], zv[kGnMaxVec];
#pragma unroll
    for (int j = 0; j < kGnMaxVec; ++j) {
        const int v = t + j * kGnThreads;
        if (v < nv) {
            yv[j] = y[v];
            zv[j] = z[v];
        }
    }
    float g[kGnMaxVec][8];  // the gated values
#pragma unroll
    for (int j = 0; j < kGnMaxVec; ++j) {
        const int v = t + j * kGnThreads;
        if (v < nv) {
            const uint32_t yw[4] = {yv[j].x, yv[j].y, yv[j].z, yv[j].w};
            const uint32_t zw[4] = {zv[j].x, zv[j].y, zv[j].z, zv[j].w};
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 yf = tc::unpack_bf16(yw[e]), zf = tc::unpack_bf16(zw[e]);
                g[j][2 * e] = yf.x * silu_fast(zf.x);
                g[j][2 * e + 1] = yf.y * silu_fast(zf.y);
                s = fmaf(g[j][2 * e], g[j][2 * e], s);
                s = fmaf(g[j][2 * e + 1], g[j][2 * e + 1], s);
            }
            ss_vec[v] = s;
        }
    }
    __syncthreads();
    for (int gi = warp; gi < ng; gi += kGnThreads / 32) {
        float s = 0.f;
        for (int v = gi * gv + lane; v < (gi + 1) * gv; v += 32) s += ss_vec[v];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) scale[gi] = rsqrtf(s / (float)a.group + a.eps);
    }
    __syncthreads();
    uint4 *out = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + row);
    const float4 *w4 = reinterpret_cast<const float4 *>(a.w);
#pragma unroll
    for (int j = 0; j < kGnMaxVec; ++j) {
        const int v = t + j * kGnThreads;
        if (v < nv) {
            const float f = scale[v / gv];
            const float4 wa = w4[2 * v], wb = w4[2 * v + 1];
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[e] = tc::pack_bf16(g[j][2 * e] * f * wv[2 * e], g[j][2 * e + 1] * f * wv[2 * e + 1]);
            out[v] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace

bool gate_norm_supported(const GateNormArgs &a)
{
    return a.M > 0 && a.C > 0 && a.group > 0 && a.C % a.group == 0 && a.group % 8 == 0 &&
           a.C <= 8 * kGnMaxVec * kGnThreads;
}

cudaError_t launch_gate_norm(const GateNormArgs &a, cudaStream_t s)
{
    Phase ph(MATE_PHASE_GATE_NORM, s);
    gate_norm_kernel<<<a.M, kGnThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace mate
