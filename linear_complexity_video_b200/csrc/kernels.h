// Launch-side view of the MATE kernels: argument blocks filled by the C ABI
// layer (mate_abi.cu) and the launchers each kernel file provides.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mate {

// Division of non-negative 32-bit integers below 2^31 by a divisor fixed at
// launch (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", PLDI 1994, figure 4.1): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (mulhi(m, n) + n) >> l. Three
// integer instructions instead of a general division.
struct FastDiv {
    uint32_t d, m, l;
};

inline FastDiv make_fastdiv(uint32_t d)
{
    FastDiv f;
    f.d = d;
    f.l = 0;
    while (f.l < 31 && (1u << f.l) < d) ++f.l;
    f.m = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << f.l) - d)) / d + 1);
    return f;
}

#ifdef __CUDACC__
__host__ __device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f)
{
#ifdef __CUDA_ARCH__
    const uint32_t hi = __umulhi(n, f.m);
#else
    const uint32_t hi = (uint32_t)(((uint64_t)n * f.m) >> 32);
#endif
    return (hi + n) >> f.l;
}
#endif

// Everything one bi-SSD call needs, resolved on the host.
struct SsdArgs {
    const void *x;
    const float *dt;
    const float *A;
    const void *B;
    const void *C;
    const float *D;
    void *out;
    int batch, T, H, W, N;   // grid; N = T*H*W tokens per batch element
    int nh, P, Ns, G;        // heads, head dim, state size, B/C groups
    int Q, nchunks;          // chunk length and chunk count of the scan
    int mode;                // MATE_SCAN_*
    int dirs;                // MATE_DIR_* bit mask (1 forward, 2 flipped)
    int review;              // 1 when a review prefix precedes the scan
    int pt, ph, pw;          // review pooling box
    int Tp, Hp, Wp, Np;      // pooled grid and its token count
    int pool_splits;         // each pooling box is summed in this many parts
    int bf16;                // 1: x, B, C, out are bf16; 0: fp32
    // the same divisors for the RMS index map and the review cells, as FastDiv
    FastDiv dT, dH, dW, dHW, dpt, dph, dpw;
    // workspace carve-outs (fp32)
    float *states_f;         // (batch, nh, nchunks, P, Ns): chunk-local forward states,
                             //   overwritten by the state entering each chunk (the
                             //   tensor-core path stores them as bf16)
    float *states_b;         // same for the flipped scan
    float *alpha;            // (batch, nh, nchunks): exp(A * sum of dt over the chunk)
    float *h_init;           // (kHinitParts, batch, nh, P, Ns): state after the review prefix;
                             //   the tensor-core path writes it as parts over ranges of
                             //   review cells that the state chain adds up, the CUDA-core
                             //   path writes part 0 whole
    float *pooled;           // (batch, pool_splits, Np, nh*P + nh + G*Ns): partial box sums of x, dt, B
    float *dt_scan;          // (batch, nh, nchunks * Q): dt in scan order, zero past the sequence
                             //   end; written by the tensor-core chunk_state for chunk_out
    int *err;                // device error word (MATE_ERR_* set by bounded waits)
};

constexpr int kHinitParts = 4;

struct TesaArgs {
    const void *q;
    const void *k;
    const void *v;
    void *out;
    int batch, T, H, W, N;
    int nh, d;
    int Tw, Sw;
    int st, sh, sw;          // shifts
    int offt, offh, offw;    // window offsets (S - s) % S
    int nwt, nwh, nww;       // windows per axis
    int bf16;
    int *err;                // device error word
};

// MATE composition: out (M x N) = y1 (M x K1) w1^T + y2 (M x K2) w2^T, bf16
// row-major, w1 (N x K1) and w2 (N x K2) in the nn.Linear layout.
struct ComposeArgs {
    const void *y1, *y2, *w1, *w2;
    void *out;
    int M, N, K1, K2;
    int phase;               // MATE_PHASE_* reported for the launch (0: MATE_PHASE_COMPOSE)
    int *err;                // device error word
};

// MA-branch front-end (mate_frontend_fwd): in_proj, causal conv along the scan
// order, SiLU, softplus(dt + bias). dc = d_inner + 2 G Ns conv channels.
struct FrontArgs {
    const void *u, *w_in;                 // (batch*N, d_model), (d_inner + dc + nh, d_model) bf16
    const float *conv_w, *conv_b, *dt_bias;  // (dc, 4), (dc), (nh)
    void *z, *x, *B, *C;                  // outputs, grid order, bf16
    float *dt;                            // (batch*N, nh) fp32
    void *xbc_pre, *dt_pre;               // workspace: (batch*N, dc), (batch*N, nh) bf16
    int batch, T, H, W, N, mode;
    int d_model, d_inner, nh, G, Ns, dc;
    FastDiv dT, dH, dW, dHW;
    int *err;                             // device error word
};

// MA-branch output side (mate_gate_norm_fwd): out = y SiLU(z) / rms over each
// group of channels, times w. y, z, out: (M, C) bf16 row-major; w: (C) fp32.
struct GateNormArgs {
    const void *y, *z;
    const float *w;
    void *out;
    int M, C, group;
    float eps;
};

// Phase hook and launch counter (mate_set_phase_hook / mate_kernel_launches).
void phase_mark(int phase, int is_end, cudaStream_t s);
void count_launch();

// Brackets one phase's launch: reports it to the hook and counts the launch.
struct Phase {
    int phase;
    cudaStream_t s;
    Phase(int p, cudaStream_t st) : phase(p), s(st) { phase_mark(phase, 0, s); }
    ~Phase()
    {
        count_launch();
        phase_mark(phase, 1, s);
    }
};

// Workspace layout of a bi-SSD call; offsets in bytes from the base pointer.
struct SsdWorkspace {
    size_t states_f, states_b, alpha, h_init, pooled, dt_scan, total;
};
SsdWorkspace ssd_workspace_layout(const SsdArgs &a);

// generic CUDA-core bi-SSD path (any supported dims, fp32 or bf16)
cudaError_t launch_ssd_generic(const SsdArgs &a, cudaStream_t s);
// the generic review pooling and prefix scan for bf16, head dim 64, d_state 64
cudaError_t launch_review_bf16_64(const SsdArgs &a, cudaStream_t s);
cudaError_t launch_review_pool_bf16_64(const SsdArgs &a, cudaStream_t s);  // its two halves
cudaError_t launch_review_scan_bf16_64(const SsdArgs &a, cudaStream_t s);
// generic CUDA-core TESA path
cudaError_t launch_tesa_generic(const TesaArgs &a, cudaStream_t s);
// tensor-core TESA path (bf16, head dim 128, 128-token windows)
bool tesa_tc_supported(const TesaArgs &a);
cudaError_t launch_tesa_tc(const TesaArgs &a, cudaStream_t s);
bool compose_tc_supported(const ComposeArgs &a);
cudaError_t launch_compose_tc(const ComposeArgs &a, cudaStream_t s);
bool front_supported(const FrontArgs &a);
cudaError_t launch_front(const FrontArgs &a, cudaStream_t s);
bool gate_norm_supported(const GateNormArgs &a);
cudaError_t launch_gate_norm(const GateNormArgs &a, cudaStream_t s);
// tensor-core bi-SSD path (bf16, head dim 64, d_state 64, both directions)
bool ssd_tc_supported(const SsdArgs &a);
cudaError_t launch_ssd_tc(const SsdArgs &a, cudaStream_t s);
// debug maps
cudaError_t launch_rms_map(int T, int H, int W, int mode, int flip, int32_t *out, cudaStream_t s);
cudaError_t launch_tesa_map(const TesaArgs &a, int32_t *out, cudaStream_t s);

}  // namespace mate
