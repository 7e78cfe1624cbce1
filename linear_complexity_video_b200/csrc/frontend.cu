// MA-branch front-end: the input side of the Mamba2 block that produces the
// bi-SSD's x, B, C and dt from the block input u (paper review "LinGen ...",
// section 三, MA-Branch item 1: the branch is a bidirectional Mamba2; the pages
// name the block and its expansion factor E, and give no more of it). The
// standard Mamba2 input side is:
//   in_proj:  [z | x B C | dt_raw] = u W_in^T          (d_inner, d_inner + 2 G Ns, nh)
//   conv:     xBC_n = SiLU(b + sum_k w_k xBC_pre_{n-3+k}), causal, depthwise,
//             width 4, along the scan sequence (positions before 0 are zero)
//   dt:       softplus(dt_raw + dt_bias)
// The conv runs once, along the forward scan order, and its result feeds both
// scan directions, as the bi-SSD's inputs do. Inputs and outputs are in grid
// order; the scan order enters only through the conv's neighbour addresses.
//
// Launches: three tensor-core GEMMs (compose_tc.cu, one input part each) for z,
// the conv channels and dt_raw (bf16, the last two into the workspace), then
// one kernel for the conv and SiLU (each warp 16 scan positions x 64 channels,
// its 19 input rows loaded at once), and one for dt.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

#include <cuda_bf16.h>

#include <algorithm>

namespace mate {

namespace {

constexpr int kHalo = 3;      // conv width - 1
constexpr int kThreads = 256;

// the RMS index map with the launch-time divisors (scan position -> grid offset)
__device__ __forceinline__ int front_offset(int n, const FrontArgs &a)
{
    const uint32_t u = (uint32_t)n;
    switch (a.mode) {
    case MATE_SCAN_SR:
        return n;
    case MATE_SCAN_SC: {
        const uint32_t t = fdiv(u, a.dHW), rem = u - t * a.dHW.d;
        const uint32_t w = fdiv(rem, a.dH), hh = rem - w * a.dH.d;
        return (int)(t * a.dHW.d + hh * a.dW.d + w);
    }
    case MATE_SCAN_TR: {
        const uint32_t sp = fdiv(u, a.dT), t = u - sp * a.dT.d;
        const uint32_t hh = fdiv(sp, a.dW), w = sp - hh * a.dW.d;
        return (int)((t * a.dH.d + hh) * a.dW.d + w);
    }
    case MATE_SCAN_ZZ: {
        const uint32_t t = fdiv(u, a.dHW), rem = u - t * a.dHW.d;
        const uint32_t i = fdiv(rem, a.dW), j = rem - i * a.dW.d;
        const uint32_t hh = (t & 1) ? a.dH.d - 1 - i : i;
        const uint32_t w = ((t * a.dH.d + i) & 1) ? a.dW.d - 1 - j : j;
        return (int)((t * a.dH.d + hh) * a.dW.d + w);
    }
    default: {  // MATE_SCAN_TC
        const uint32_t sp = fdiv(u, a.dT), t = u - sp * a.dT.d;
        const uint32_t w = fdiv(sp, a.dH), hh = sp - w * a.dH.d;
        return (int)((t * a.dH.d + hh) * a.dW.d + w);
    }
    }
}

// Conv + SiLU: warp w of a CTA takes the channel pair (64 (8 blockIdx.x + w) + 2 lane,
// +1) of batch element blockIdx.z over the kWarpPos scan positions kWarpPos
// blockIdx.y ..: it loads the kWarpPos + 3 rows it needs (the halo included) with
// all loads in flight at once, then slides the width-4 window along them. For every position a
// warp reads and writes 128 contiguous bytes of a token row, and the CTA's eight
// warps cover 1 KB of it.
constexpr int kWarpPos = 16;

// SiLU of a pair, v (1 + tanh(v / 2)) / 2 with the hardware tanh (tanh.approx.f32,
// relative error about 2^-11: far below the bf16 rounding of the result)
__device__ __forceinline__ float2 silu2(float2 v)
{
    const float2 h = tc::mul_f32x2(v, make_float2(0.5f, 0.5f));
    float tx, ty;
    asm("tanh.approx.f32 %0, %1;" : "=f"(tx) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(ty) : "f"(h.y));
    return tc::fma_f32x2(h, make_float2(tx, ty), h);
}
static_assert(kWarpPos + kHalo <= 32, "one lane per input row");

__global__ void __launch_bounds__(kThreads) front_conv_kernel(FrontArgs a)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cbase = (blockIdx.x * (kThreads / 32) + warp) * 64;
    const int c = cbase + 2 * lane;
    const int s0 = blockIdx.y * kWarpPos, b = blockIdx.z;
    if (cbase >= a.dc) return;  // (a multiple of 8: whole warps past the channels leave)
    // lane i < 19 owns scan position s0 - 3 + i: its grid offset g (-1 outside the
    // sequence) and the element offset g * dc of its row of conv channels
    const int p = s0 - kHalo + lane;
    const int g_own = (lane < kWarpPos + kHalo && p >= 0 && p < a.N) ? front_offset(p, a) : -1;
    // (g * dc < 2^31: a grid holds fewer than 2^31 elements of a channel group)
    const int e_own = g_own >= 0 ? g_own * a.dc : -1;
    const bool live = c < a.dc;
    const uint32_t *pre =
        reinterpret_cast<const uint32_t *>(static_cast<const __nv_bfloat16 *>(a.xbc_pre) + (size_t)b * a.N * a.dc + c);
    uint32_t in[kWarpPos + kHalo];
#pragma unroll
    for (int i = 0; i < kWarpPos + kHalo; ++i) {
        const int e = __shfl_sync(0xffffffffu, e_own, i);
        in[i] = (e >= 0 && live) ? pre[e >> 1] : 0u;  // (e and c even: a whole bf16 pair)
    }
    // lanes past the last channel stay in the loop below (its shuffles take the whole
    // warp) but read channel 0's taps and store nothing
    const int cl = live ? c : 0;
    float2 tap[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) tap[k] = make_float2(a.conv_w[(size_t)cl * 4 + k], a.conv_w[(size_t)(cl + 1) * 4 + k]);
    const float2 bias = make_float2(a.conv_b[cl], a.conv_b[cl + 1]);
    // where this channel pair goes: x, B or C (a pair never straddles two of them)
    const int gns = a.G * a.Ns;
    __nv_bfloat16 *dst;
    int width, cofs;
    if (cl < a.d_inner) {
        dst = static_cast<__nv_bfloat16 *>(a.x), width = a.d_inner, cofs = cl;
    } else if (cl < a.d_inner + gns) {
        dst = static_cast<__nv_bfloat16 *>(a.B), width = gns, cofs = cl - a.d_inner;
    } else {
        dst = static_cast<__nv_bfloat16 *>(a.C), width = gns, cofs = cl - a.d_inner - gns;
    }
    uint32_t *out = reinterpret_cast<uint32_t *>(dst + (size_t)b * a.N * width + cofs);
    const int wpairs = width >> 1;  // bf16 pairs per token row of the destination
    // the window of rows j .. j + 3, unpacked as it slides (each row once), so that the
    // packed rows are all the registers the loads hold
    float2 w0 = tc::unpack_bf16(in[0]), w1 = tc::unpack_bf16(in[1]), w2 = tc::unpack_bf16(in[2]);
#pragma unroll
    for (int j = 0; j < kWarpPos; ++j) {
        // output position s0 + j: inputs at rows j .. j + 3
        const float2 w3 = tc::unpack_bf16(in[j + kHalo]);
        float2 v = tc::fma_f32x2(tap[0], w0, bias);
        v = tc::fma_f32x2(tap[1], w1, v);
        v = tc::fma_f32x2(tap[2], w2, v);
        v = tc::fma_f32x2(tap[3], w3, v);
        w0 = w1, w1 = w2, w2 = w3;
        const float2 y = silu2(v);
        const int g = __shfl_sync(0xffffffffu, g_own, j + kHalo);
        if (g >= 0 && live) out[g * wpairs] = tc::pack_bf16(y.x, y.y);
    }
}

// dt = softplus(dt_raw + dt_bias), grid order, fp32 out
__global__ void __launch_bounds__(kThreads) front_dt_kernel(FrontArgs a)
{
    const size_t total = (size_t)a.batch * a.N * a.nh;
    const __nv_bfloat16 *raw = static_cast<const __nv_bfloat16 *>(a.dt_pre);
    for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < total; i += (size_t)gridDim.x * kThreads) {
        const float v = __bfloat162float(raw[i]) + a.dt_bias[i % a.nh];
        a.dt[i] = v > 20.f ? v : log1pf(__expf(v));
    }
}

}  // namespace

bool front_supported(const FrontArgs &a)
{
    ComposeArgs g = {};
    g.M = a.batch * a.N;
    g.K1 = a.d_model;
    g.N = a.d_inner;
    bool ok = compose_tc_supported(g);
    g.N = a.dc;
    ok = ok && compose_tc_supported(g);
    g.N = a.nh;
    ok = ok && compose_tc_supported(g);
    return ok && a.dc % 8 == 0 && a.d_inner % 2 == 0 && (a.G * a.Ns) % 2 == 0;
}

cudaError_t launch_front(const FrontArgs &a, cudaStream_t s)
{
    const size_t M = (size_t)a.batch * a.N;
    const __nv_bfloat16 *w = static_cast<const __nv_bfloat16 *>(a.w_in);
    // in_proj, one output group per GEMM: rows [0, d_inner) of W_in -> z, the next dc
    // rows -> the conv's inputs, the last nh rows -> dt_raw
    const void *outs[3] = {a.z, a.xbc_pre, a.dt_pre};
    const int ns[3] = {a.d_inner, a.dc, a.nh};
    size_t row0 = 0;
    for (int i = 0; i < 3; ++i) {
        ComposeArgs g = {};
        g.y1 = a.u;
        g.w1 = w + row0 * a.d_model;
        g.y2 = nullptr;
        g.w2 = nullptr;
        g.out = const_cast<void *>(outs[i]);
        g.M = (int)M;
        g.N = ns[i];
        g.K1 = a.d_model;
        g.K2 = 0;
        g.phase = MATE_PHASE_FRONT_PROJ;
        g.err = a.err;
        cudaError_t e = launch_compose_tc(g, s);
        if (e != cudaSuccess) return e;
        row0 += ns[i];
    }
    {
        Phase ph(MATE_PHASE_FRONT_CONV, s);
        front_conv_kernel<<<dim3((a.dc + 64 * (kThreads / 32) - 1) / (64 * (kThreads / 32)),
                                 (a.N + kWarpPos - 1) / kWarpPos, a.batch),
                            kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    {
        Phase ph(MATE_PHASE_FRONT_DT, s);
        const size_t total = M * a.nh;
        const int blocks = (int)std::min<size_t>((total + kThreads - 1) / kThreads, 148 * 8);
        front_dt_kernel<<<blocks, kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace mate
