/*
 * mate.h - C ABI of the MATE token-mix library (libmate.so) for NVIDIA B200
 * (sm_100a).
 *
 * The library computes the token-mixing core of LinGen's MATE block, the
 * linear-complexity block that replaces DiT self-attention:
 *   - the MA-branch: a bidirectional Mamba2 (SSD) selective scan over the
 *     T x H x W latent token grid, unrolled in one of the four Rotary Major
 *     Scan orders, optionally preceded by review tokens;
 *   - the TE-branch: TEmporal Swin Attention (TESA), softmax attention inside
 *     fixed Tw x Sw x Sw windows whose placement is shifted on alternate
 *     layers.
 * Sources: "LinGen: Towards High-Resolution Minute-Length Text-to-Video
 * Generation with Linear Computational Complexity" (xllm-io paper review),
 * section 三 "技术架构", MA-Branch items 1-3 and TE-Branch; the QbitAI news
 * article on LinGen, method section.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller. The
 *     library allocates no device memory and keeps no state between calls,
 *     with two exceptions that are part of its device image: one device-side
 *     error word (see mate_last_error) and the fixed scratch array of
 *     mate_bissd_fwd_noalloc (MATE_NOALLOC_SCRATCH_BYTES, below).
 *   - Storage type decides which kernels run, with no fallback between them:
 *     bf16 tensors run on the tensor-core (tcgen05) kernels, fp32 tensors on
 *     the CUDA-core kernels. A bf16 call whose dims the tensor-core kernels
 *     do not take returns MATE_ERR_UNSUPPORTED.
 *   - The library caches, per device, the device addresses of its own device
 *     variables. Destroying a device's primary context (cudaDeviceReset) is
 *     detected through the context's unique id, and the addresses are looked
 *     up again on the next call.
 *   - Tensors are dense and contiguous in grid order: for a batch element,
 *     token (t, h, w) sits at grid offset (t*H + h)*W + w, W fastest.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued on it; calls return before it finishes.
 *   - Inputs are never written. Outputs must not overlap any input.
 *   - Return value: MATE_OK, or a negative MATE_ERR_* code. Argument errors
 *     are detected on the host before anything is enqueued; nothing is
 *     written then.
 */
#ifndef MATE_H
#define MATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define MATE_OK 0
#define MATE_ERR_INVALID_ARG (-1) /* null or misaligned pointer, bad size, overlap  */
#define MATE_ERR_UNSUPPORTED (-2) /* dims or dtype outside the compiled set          */
#define MATE_ERR_CUDA (-3)        /* a CUDA launch or runtime call failed            */
#define MATE_ERR_TIMEOUT (-4)     /* a bounded device-side wait gave up              */
#define MATE_ERR_WORKSPACE (-5)   /* workspace missing, too small or misaligned      */

/* ---- element types ------------------------------------------------------ */
#define MATE_F32 0  /* x, B, C, q, k, v, out stored as IEEE fp32 */
#define MATE_BF16 1 /* x, B, C, q, k, v, out stored as bf16; fp32 accumulation */

/* ---- Rotary Major Scan orders (paper review, MA-Branch item 2) ----------
 * Scan position n of a T x H x W grid maps to these grid coordinates:
 *   SR spatial-row:     n = (t*H + h)*W + w      (W fastest, then H, then T)
 *   SC spatial-column:  n = (t*W + w)*H + h      (H fastest, then W, then T)
 *   TR temporal-row:    n = (h*W + w)*T + t      (T fastest, then W, then H)
 *   TC temporal-column: n = (w*H + h)*T + t      (T fastest, then H, then W)
 * The QbitAI article gives W, H, T the first, second and third priority in
 * its example and obtains the other scans by exchanging priorities; "row"
 * puts W before H, "temporal" puts T first. The flipped scan visits
 * position N-1-n at step n (the review prints this as T*H*W - n with n
 * counted from 1). */
#define MATE_SCAN_SR 0
#define MATE_SCAN_SC 1
#define MATE_SCAN_TR 2
#define MATE_SCAN_TC 3
/* Zigzag scan, the alternative the pages compare RMS against (QbitAI article,
 * method section; paper review, 5.5 Table 2: "Zigzag ... 144 s"). The pages
 * do not define it; it is read here as the 3D boustrophedon in which every
 * step moves to a neighbouring token: frames in time order, the rows of even
 * frames top to bottom and of odd frames bottom to top, and global row
 * R = t*H + i (i = row counted in visiting order) walked along W left to
 * right when R is even, right to left when R is odd:
 *   n = (t*H + i)*W + j,  h = t even ? i : H-1-i,  w = R even ? j : W-1-j.
 * Its sub-chunks are not boxes of the grid, so the kernels gather its rows.
 * The flipped scan is defined as for the RMS orders. */
#define MATE_SCAN_ZZ 4

/* directions of the bidirectional scan (test and diagnosis aid) */
#define MATE_DIR_FWD 1 /* the scan in RMS order only          */
#define MATE_DIR_BWD 2 /* the flipped scan only, flipped back */
#define MATE_DIR_BI 3  /* their sum (the MA-branch output)    */

typedef struct {
    int batch;      /* batch elements, >= 1                                  */
    int nheads;     /* SSD heads nh                                          */
    int headdim;    /* head dimension P                                      */
    int dstate;     /* state size Ns (d_state)                               */
    int ngroups;    /* B/C groups G; head h reads group h / (nh / G)         */
    int chunk;      /* scan chunk length Q, a tiling choice: outputs do not  */
                    /* depend on it beyond rounding                          */
    int dtype;      /* MATE_F32 or MATE_BF16                                 */
    int directions; /* MATE_DIR_*; 0 means MATE_DIR_BI                       */
} mate_ssd_dims;

typedef struct {
    int batch;   /* batch elements, >= 1   */
    int nheads;  /* attention heads        */
    int headdim; /* head dimension d       */
    int dtype;   /* MATE_F32 or MATE_BF16  */
} mate_attn_dims;

/*
 * Workspace bytes mate_bissd_fwd needs for these dims (0 on bad or
 * unsupported arguments, which mate_bissd_fwd then reports). The workspace
 * holds per-chunk scan states of both directions (bf16 for bf16 storage,
 * fp32 for fp32 storage), chunk decays, for bf16 storage dt in scan order
 * (fp32, one value per head and scan position, padded to whole chunks) and,
 * with review tokens, the pooled grid and the state the review prefix
 * leaves behind. Its contents on entry
 * do not matter. It grows linearly with batch * T * H * W * nheads / chunk.
 */
size_t mate_bissd_workspace_bytes(int T, int H, int W, const int review_pool[3], const mate_ssd_dims *d);

/*
 * MA-branch token mix: bidirectional Mamba2 / SSD scan in Rotary Major Scan
 * order with optional review tokens (paper review, MA-Branch items 1-3).
 *
 * For each batch element and head h, let X be the grid unrolled in scan
 * order `scan_mode` (MATE_SCAN_SR .. MATE_SCAN_TC, or MATE_SCAN_ZZ for the
 * zigzag comparison; N = T*H*W tokens). With state s (headdim x dstate,
 * zero at the start of every scanned sequence) the scan computes
 *     s_n = exp(dt_n * A[h]) * s_{n-1} + dt_n * x_n B_n^T
 *     y_n = s_n C_n + D[h] * x_n
 * once over [prefix, X] and once over [prefix, flip(X)]. The outputs at
 * prefix positions are dropped, the second result is flipped back, and the
 * two are added: out = y_forward + y_flipped (so D*x enters twice).
 *
 * Review tokens (review_pool = {pt, ph, pw}, all > 0 and dividing T, H, W):
 * x, dt and B are average-pooled over non-overlapping pt x ph x pw boxes,
 * the pooled grid is unrolled in the same scan order into R, and the prefix
 * is [R, flip(R)] (2*T*H*W/(pt*ph*pw) tokens). That prefix reads the same
 * forwards and backwards, so it precedes both scans unchanged. Outputs at
 * prefix positions are dropped, so pooled C would never be used and is not
 * computed. review_pool NULL or {0, 0, 0}: no prefix.
 *
 * Layouts (contiguous, grid order):
 *   x, out : (batch, T, H, W, nheads, headdim)   dtype
 *   dt     : (batch, T, H, W, nheads)            fp32, > 0 expected
 *   A, D   : (nheads)                            fp32 (A < 0 expected)
 *   B, C   : (batch, T, H, W, ngroups, dstate)   dtype
 * x, B, C and out must be 16-byte aligned; dt, A, D 4-byte aligned.
 * workspace: >= mate_bissd_workspace_bytes(...) bytes of device memory,
 *   256-byte aligned, used only by the work this call enqueues.
 * Supported (nheads % ngroups == 0 and T*H*W < 2^31 throughout):
 *   bf16 storage (tensor-core kernels): headdim = dstate = 64, chunk a
 *     multiple of 128 in [128, 512], directions = MATE_DIR_BI;
 *   fp32 storage (CUDA-core kernels): headdim and dstate in {16, 32, 64},
 *     chunk in [1, 256], any directions.
 *   Anything else returns MATE_ERR_UNSUPPORTED before enqueueing work.
 * Reproducibility: with review tokens on the tensor-core path, the review
 *   box sums are accumulated with floating-point atomics, so the bits of
 *   the result can differ from run to run (the differences are rounding
 *   level, far inside the stated tolerance). Without review tokens, and on
 *   the CUDA-core path, results are bitwise reproducible.
 * Returns MATE_OK, MATE_ERR_INVALID_ARG, MATE_ERR_UNSUPPORTED,
 *   MATE_ERR_WORKSPACE or MATE_ERR_CUDA.
 */
int mate_bissd_fwd(const void *x, const float *dt, const float *A, const void *B, const void *C,
                   const float *D, int T, int H, int W, int scan_mode, const int review_pool[3],
                   void *out, const mate_ssd_dims *d, void *workspace, size_t ws_bytes, void *stream);

/*
 * Allocation-free variant of mate_bissd_fwd. The paper has no counterpart:
 * this is a deployment aid of this library.
 *
 * Who needs it: callers that cannot allocate device memory on their call
 * path, such as a plugin inside a host application that owns the whole
 * device memory pool, code that must not pay the implicit device
 * synchronisation of cudaMalloc/cudaFree, or a process whose device memory
 * budget is fixed up front. They pass inputs and outputs only; the scratch
 * that mate_bissd_fwd takes as `workspace` comes from a fixed array of
 * MATE_NOALLOC_SCRATCH_BYTES bytes that is part of the library's device
 * image. Every GPU that loads the library holds that array until the
 * process exits.
 *
 * Arguments, layouts and results are those of mate_bissd_fwd.
 * - Returns MATE_ERR_WORKSPACE, enqueueing nothing, when
 *   mate_bissd_workspace_bytes(...) for these dims exceeds
 *   MATE_NOALLOC_SCRATCH_BYTES.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture. The first call after the device's primary
 *   context was destroyed and re-created looks it up again.
 * - All calls share the one array, which keeps the last call's contents.
 *   Calls whose work may overlap on the GPU (e.g. on unordered streams) race
 *   on it and must be serialised by the caller. Nothing needs clearing
 *   between calls: the kernels write every scratch word before reading it.
 * - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define MATE_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */
int mate_bissd_fwd_noalloc(const void *x, const float *dt, const float *A, const void *B, const void *C,
                           const float *D, int T, int H, int W, int scan_mode, const int review_pool[3],
                           void *out, const mate_ssd_dims *d, void *stream);

/*
 * TE-branch: TEmporal Swin Attention (paper review, TE-Branch; the superapi
 * product page, "Technical Principles": windows shift between layers).
 *
 * The grid is cut into windows of Tw x Sw x Sw tokens. Along each axis the
 * window boundaries sit at the coordinates congruent to that axis' shift
 * modulo the window size (shift = {st, sh, sw}, 0 <= st < Tw,
 * 0 <= sh, sw < Sw), so with a non-zero shift the first and last window
 * along that axis are partial. This is the same partition as rolling the
 * grid by the shift and masking wrapped-around pairs. Each token attends to
 * the tokens of its own window only, per head:
 *     out_i = sum_j softmax_j(q_i . k_j / sqrt(headdim)) v_j
 * with no mask inside a window and no position bias.
 *
 * Layouts: q, k, v, out : (batch, T, H, W, nheads, headdim), dtype,
 *   16-byte aligned.
 * Supported:
 *   bf16 storage (tensor-core kernel): headdim = 128, Tw*Sw*Sw = 128;
 *   fp32 storage (CUDA-core kernel): headdim in {16, 32, 64, 128},
 *     Tw*Sw*Sw <= 512.
 *   Anything else returns MATE_ERR_UNSUPPORTED.
 * Returns MATE_OK, MATE_ERR_INVALID_ARG, MATE_ERR_UNSUPPORTED or
 *   MATE_ERR_CUDA.
 */
int tesa_fwd(const void *q, const void *k, const void *v, int T, int H, int W, int Tw, int Sw,
             const int shift[3], void *out, const mate_attn_dims *d, void *stream);

/* ---- MATE composition ---------------------------------------------------- */
typedef struct {
    int tokens;  /* rows M of every operand (all batch elements, grid order) */
    int k_ma;    /* MA-branch channels (SSD heads x head dim, e.g. 80 x 64) */
    int k_te;    /* TE-branch channels (TESA heads x head dim, e.g. 20 x 128) */
    int d_model; /* output channels N (the block width, e.g. 2560) */
    int dtype;   /* MATE_BF16 (the only storage the kernel takes) */
} mate_compose_dims;

/*
 * MATE composition (paper review, section 三, MATE: the MA-branch and the
 * TE-branch together replace self-attention). The pages give no combination
 * rule; the two branch outputs have different widths, so each is projected
 * to the model width and the projections are added:
 *     out = y_ma W_ma^T + y_te W_te^T
 * computed as one bf16 tensor-core GEMM over the concatenated K_MA + K_TE
 * reduction with fp32 accumulation, rounded once to bf16.
 *   y_ma : (tokens, k_ma)     bf16, row-major (the bi-SSD output viewed as rows)
 *   y_te : (tokens, k_te)     bf16, row-major (the TESA output viewed as rows)
 *   w_ma : (d_model, k_ma)    bf16, row-major (nn.Linear layout)
 *   w_te : (d_model, k_te)    bf16, row-major
 *   out  : (tokens, d_model)  bf16, row-major, caller-owned, must not overlap
 *          the inputs
 * All pointers device memory, 16-byte aligned. k_ma and k_te are multiples of
 * 64 (either may be 0, not both), d_model a multiple of 64, tokens > 0.
 * Returns MATE_OK, MATE_ERR_INVALID_ARG (bad pointers, sizes or overlap),
 * MATE_ERR_UNSUPPORTED (other dtype or sizes) or MATE_ERR_CUDA.
 */
int mate_compose_fwd(const void *y_ma, const void *y_te, const void *w_ma, const void *w_te, void *out,
                     const mate_compose_dims *d, void *stream);

/* ---- MA-branch output side ----------------------------------------------- */
typedef struct {
    int tokens;   /* rows */
    int channels; /* C = d_inner of the bi-SSD (nheads * headdim, e.g. 5120) */
    int group;    /* channels per norm group (Mamba2: d_inner / ngroups)       */
    int dtype;    /* MATE_BF16 (the only storage the kernel takes)             */
} mate_gate_norm_dims;

/*
 * MA-branch output side (paper review, section 三, MA-Branch item 1, the
 * bidirectional Mamba2 block; the pages give no more of it, so this is the
 * standard Mamba2 gated RMS norm, gate first): per row and group of `group`
 * consecutive channels,
 *     v_k   = y_k SiLU(z_k)
 *     out_k = v_k w_k / sqrt(mean_{k in group} v_k^2 + eps)
 * in fp32, rounded once to bf16. Its output is the MA-branch's input to
 * mate_compose_fwd.
 *   y   : (tokens, channels) bf16, row-major (the bi-SSD output viewed as rows)
 *   z   : (tokens, channels) bf16, row-major (mate_frontend_fwd's z)
 *   w   : (channels)         fp32, the norm weight
 *   out : (tokens, channels) bf16, row-major, caller-owned, must not overlap
 *         y, z or w
 * All pointers device memory, 16-byte aligned; eps >= 0 and finite. group a
 * multiple of 8 that divides channels, channels <= 8192, tokens > 0.
 * Returns MATE_OK, MATE_ERR_INVALID_ARG (bad pointers, sizes, eps or overlap),
 * MATE_ERR_UNSUPPORTED (other dtype or sizes) or MATE_ERR_CUDA.
 */
int mate_gate_norm_fwd(const void *y, const void *z, const float *w, float eps, void *out,
                       const mate_gate_norm_dims *d, void *stream);

/* ---- MA-branch front-end ------------------------------------------------- */
typedef struct {
    int batch;
    int d_model; /* block width (e.g. 2560) */
    int nheads;  /* SSD heads; d_inner = nheads * headdim (e.g. 80 x 64) */
    int headdim;
    int ngroups; /* B/C groups */
    int dstate;
    int dtype;   /* MATE_BF16 (the only storage the kernels take) */
} mate_frontend_dims;

/*
 * Workspace bytes mate_frontend_fwd needs (0 on bad or unsupported
 * arguments): the in_proj outputs that the conv and dt steps read, bf16.
 */
size_t mate_frontend_workspace_bytes(int T, int H, int W, const mate_frontend_dims *d);

/*
 * MA-branch front-end: the input side of the Mamba2 block that produces the
 * bi-SSD's inputs (paper review, section 三, MA-Branch item 1, bidirectional
 * Mamba2; the pages give no more of the block, so this is the standard
 * Mamba2 input side, with d_inner = nheads * headdim and dc = d_inner + 2 *
 * ngroups * dstate conv channels):
 *     [z | xBC_pre | dt_raw] = u W_in^T
 *     xBC_n = SiLU(conv_b + sum_{k=0..3} conv_w[., k] * xBC_pre_{n-3+k})
 *             along the scan order `scan_mode` (causal, depthwise, width 4,
 *             positions before the first are zero); xBC = [x | B | C]
 *     dt = softplus(dt_raw + dt_bias)
 * The conv runs once, in the forward scan order; its result feeds both scan
 * directions of mate_bissd_fwd. Everything stays in grid order.
 *   u      : (batch, T, H, W, d_model)              bf16
 *   w_in   : (d_inner + dc + nheads, d_model)       bf16 (nn.Linear layout,
 *            rows z, then x, B, C, then dt)
 *   conv_w : (dc, 4) fp32;  conv_b : (dc) fp32;  dt_bias : (nheads) fp32
 *   z      : (batch, T, H, W, d_inner)              bf16 (the gate of mate_gate_norm_fwd)
 *   x      : (batch, T, H, W, nheads, headdim)      bf16
 *   dt     : (batch, T, H, W, nheads)               fp32
 *   B, C   : (batch, T, H, W, ngroups, dstate)      bf16
 * Device pointers; bf16 ones 16-byte aligned, fp32 ones 4-byte aligned;
 * outputs caller-owned and disjoint from the inputs and the workspace.
 * Supported: d_model a multiple of 64, d_inner and ngroups * dstate even,
 * dc and nheads multiples of 8, T*H*W * dc < 2^31. Returns MATE_OK, MATE_ERR_INVALID_ARG,
 * MATE_ERR_UNSUPPORTED, MATE_ERR_WORKSPACE or MATE_ERR_CUDA.
 */
int mate_frontend_fwd(const void *u, const void *w_in, const float *conv_w, const float *conv_b, const float *dt_bias,
                      int T, int H, int W, int scan_mode, void *z, void *x, float *dt, void *B, void *C,
                      const mate_frontend_dims *d, void *workspace, size_t ws_bytes, void *stream);

/*
 * Debug export of the scan order the kernels use: out_dev[n] = grid offset
 * of the n-th token of the scan (flip != 0: of the flipped scan). out_dev
 * holds T*H*W int32 (device memory, caller-owned).
 */
int mate_debug_rms_map(int T, int H, int W, int scan_mode, int flip, int32_t *out_dev, void *stream);

/*
 * Test hook for the integer division the tensor-core SSD kernels use for the
 * scan-order index map and the review cells (a divisor fixed per call,
 * multiply-high form; no counterpart in the pages): q[i] = n[i] / d for
 * count values, computed on the host with the same code the kernels run.
 * n and q are host arrays (caller-owned); every n[i] must be below 2^31 and
 * 1 <= d < 2^31. Returns MATE_OK, or MATE_ERR_INVALID_ARG (nothing written)
 * for null arrays or values out of range.
 */
int mate_debug_fastdiv(const uint32_t *n, uint32_t *q, size_t count, uint32_t d);

/*
 * Debug export of the TESA window partition the kernels use: out_win_dev[g]
 * = window id of grid token g, windows numbered in (t, h, w) order of their
 * first token. out_win_dev holds T*H*W int32 (device memory, caller-owned).
 */
int mate_debug_tesa_map(int T, int H, int W, int Tw, int Sw, const int shift[3], int32_t *out_win_dev,
                        void *stream);

/*
 * Synchronises `stream`, then returns and clears the device-side error word
 * that kernels set when a bounded wait gives up (MATE_ERR_TIMEOUT) or a
 * device-side check fails (MATE_ERR_INVALID_ARG). Returns MATE_ERR_CUDA if
 * the synchronisation itself fails.
 */
int mate_last_error(void *stream);

/*
 * Phases of a call, reported to the phase hook below. Each phase is one
 * kernel launch, or (REVIEW_POOL when CHUNK_STATE takes the box sums, which
 * it does when a review box is 4 or 8 tokens long on the scan's fastest axis
 * on the tensor-core path) one clearing of the box-sum buffer.
 */
#define MATE_PHASE_REVIEW_POOL 1 /* box sums of x, dt, B over the review boxes     */
#define MATE_PHASE_REVIEW_SCAN 2 /* the state the review prefix leaves (h_init)    */
#define MATE_PHASE_CHUNK_STATE 3 /* chunk-local scan states (and box sums, above)  */
#define MATE_PHASE_STATE_PASS 4  /* chain chunk states -> state entering each chunk */
#define MATE_PHASE_CHUNK_OUT 5   /* outputs of every chunk, both directions         */
#define MATE_PHASE_TESA 6        /* windowed attention                             */
#define MATE_PHASE_COMPOSE 7     /* mate_compose_fwd's projection GEMM              */
#define MATE_PHASE_FRONT_PROJ 8  /* mate_frontend_fwd: one in_proj GEMM (3 per call) */
#define MATE_PHASE_FRONT_CONV 9  /* mate_frontend_fwd: conv along the scan + SiLU   */
#define MATE_PHASE_FRONT_DT 10   /* mate_frontend_fwd: softplus(dt + bias)          */
#define MATE_PHASE_GATE_NORM 11  /* mate_gate_norm_fwd                              */

/*
 * Optional enqueue-time hook, for timing phases with events on the caller's
 * stream: while set, the library calls fn(phase, is_end, stream, user) on the
 * calling host thread right before (is_end = 0) and right after (is_end = 1)
 * it enqueues each phase on `stream`. NULL removes the hook. Process-wide;
 * set or clear it only while no other thread is calling into the library.
 */
typedef void (*mate_phase_hook)(int phase, int is_end, void *stream, void *user);
void mate_set_phase_hook(mate_phase_hook fn, void *user);

/* Number of kernels the library has launched since the process started. */
uint64_t mate_kernel_launches(void);

/* Static text for a status code. */
const char *mate_status_string(int code);

/* Library version, major*10000 + minor*100 + patch. */
int mate_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MATE_H */
