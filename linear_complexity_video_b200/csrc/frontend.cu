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
// one kernel for the conv and SiLU over 128 scan positions x 128 channels per
// CTA (rows staged in shared memory with their 3-position halo), and one for dt.
#include "common.cuh"
#include "kernels.h"

#include <cuda_bf16.h>

#include <algorithm>

namespace mate {

namespace {

constexpr int kPos = 128;     // scan positions per CTA
constexpr int kCh = 128;      // conv channels per CTA
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

// Conv + SiLU for scan positions [s0, s0 + 128) and channels [c0, c0 + 128) of
// batch element b. Thread t takes the channel pair (c0 + 2 (t % 64), +1) over the
// 32 positions 32 (t / 64) .. and slides the width-4 window along them.
__global__ void __launch_bounds__(kThreads) front_conv_kernel(FrontArgs a)
{
    __shared__ __align__(16) __nv_bfloat16 rows[kPos + kHalo][kCh];
    __shared__ int goff[kPos];
    const int tid = threadIdx.x;
    const int s0 = blockIdx.x * kPos, c0 = blockIdx.y * kCh, b = blockIdx.z;
    const int nch = min(kCh, a.dc - c0);  // channels of this CTA (a multiple of 8)
    // grid offsets of the 128 output positions
    for (int i = tid; i < kPos; i += kThreads) goff[i] = s0 + i < a.N ? front_offset(s0 + i, a) : 0;
    // the 131 input rows (positions s0 - 3 ..), 16 bytes per request, zeros outside the sequence
    const __nv_bfloat16 *pre = static_cast<const __nv_bfloat16 *>(a.xbc_pre);
    for (int q = tid; q < (kPos + kHalo) * (kCh / 8); q += kThreads) {
        const int i = q / (kCh / 8), cc = (q % (kCh / 8)) * 8;
        const int p = s0 - kHalo + i;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (p >= 0 && p < a.N && cc < nch) {
            const int g = front_offset(p, a);
            v = *reinterpret_cast<const uint4 *>(pre + ((size_t)b * a.N + g) * a.dc + c0 + cc);
        }
        *reinterpret_cast<uint4 *>(&rows[i][cc]) = v;
    }
    __syncthreads();
    const int cp = 2 * (tid % 64), pg = tid / 64;
    if (cp >= nch) return;
    const int c = c0 + cp;
    float w0[4], w1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        w0[k] = a.conv_w[(size_t)c * 4 + k];
        w1[k] = a.conv_w[(size_t)(c + 1) * 4 + k];
    }
    const float b0 = a.conv_b[c], b1 = a.conv_b[c + 1];
    // where this channel pair goes: x, B or C (a pair never straddles two of them)
    const int gns = a.G * a.Ns;
    __nv_bfloat16 *dst;
    int width, cofs;
    if (c < a.d_inner) {
        dst = static_cast<__nv_bfloat16 *>(a.x), width = a.d_inner, cofs = c;
    } else if (c < a.d_inner + gns) {
        dst = static_cast<__nv_bfloat16 *>(a.B), width = gns, cofs = c - a.d_inner;
    } else {
        dst = static_cast<__nv_bfloat16 *>(a.C), width = gns, cofs = c - a.d_inner - gns;
    }
    // the window: inputs at positions n-3, n-2, n-1 of the first output n = 32 pg
    float2 in[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) in[k] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&rows[32 * pg + k][cp]));
    for (int j = 0; j < 32; ++j) {
        const int i = 32 * pg + j;  // output position s0 + i sits at row i + 3
        const float2 cur = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&rows[i + kHalo][cp]));
        float v0 = b0 + w0[0] * in[0].x + w0[1] * in[1].x + w0[2] * in[2].x + w0[3] * cur.x;
        float v1 = b1 + w1[0] * in[0].y + w1[1] * in[1].y + w1[2] * in[2].y + w1[3] * cur.y;
        v0 = v0 / (1.f + __expf(-v0));  // SiLU
        v1 = v1 / (1.f + __expf(-v1));
        if (s0 + i < a.N)
            *reinterpret_cast<__nv_bfloat162 *>(dst + ((size_t)b * a.N + goff[i]) * width + cofs) =
                __floats2bfloat162_rn(v0, v1);
        in[0] = in[1];
        in[1] = in[2];
        in[2] = cur;
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
        front_conv_kernel<<<dim3((a.N + kPos - 1) / kPos, (a.dc + kCh - 1) / kCh, a.batch), kThreads, 0, s>>>(a);
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
