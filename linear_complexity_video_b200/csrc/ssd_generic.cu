// Bidirectional Mamba2 (SSD) scan in Rotary Major Scan order with review
// tokens: CUDA-core path for fp32 storage and any supported head size (bf16
// storage runs on the tensor-core kernels of ssd_tc.cu). The review pooling
// kernels here also serve the tensor-core path.
//
// Method (paper review "LinGen ...", section 三, MA-Branch items 1-3): per
// head, s_n = exp(dt_n A) s_{n-1} + dt_n x_n B_n^T and y_n = s_n C_n + D x_n,
// scanned over the RMS-ordered sequence and over its flip; the flipped
// outputs are flipped back and added. Review tokens prepend a pooled copy of
// the grid and its flip.
//
// Decomposition (the chunked "state-space duality" form of Mamba2). The
// sequence is cut into chunks of Q tokens. Inside a chunk, with
// cum_i = A * sum_{k<=i} dt_k and excl_i = cum_i - A dt_i (both from the
// chunk start), the forward direction contributes
//     sum_{j<=i} (C_i.B_j) exp(cum_i - cum_j) dt_j x_j + exp(cum_i) C_i S_in
// and the flipped direction, written in original order,
//     sum_{j>=i} (C_i.B_j) exp(excl_j - excl_i) dt_j x_j + exp(cum_end - excl_i) C_i S'_in
// where S_in is the forward state entering the chunk from the left and S'_in
// the flipped-scan state entering it from the right. The review prefix reads
// the same in both directions, so both scans start from the one state it
// leaves behind (h_init).
//
// Kernels:
//   review_pool   average-pool x, dt, B over each pooling box
//   review_scan   scan the prefix [R, flip(R)] from zero -> h_init
//   chunk_state   chunk-local forward and flipped states and chunk decay
//   state_pass    chain the chunk states: state entering every chunk
//   chunk_out     intra-chunk quadratic term + entering states + D x
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace mate {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;
constexpr int kMaxStateChunk = 1024;  // chunk_state handles chunks of up to this many tokens

__device__ __forceinline__ size_t tok_index(const SsdArgs &a, int b, int g) { return (size_t)b * a.N + g; }

// ---------------------------------------------------------------------------
// review_pool: pooled[b][s][cell][ch] = sum of x | dt | B over part s of the
// cell's box (the box's tokens, row-major, cut into pool_splits ranges).
// grid: (Np, ceil(channels / 256), batch * pool_splits)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void split_range(int box, int splits, int s, int &lo, int &hi)
{
    lo = (int)(((long long)box * s) / splits);
    hi = (int)(((long long)box * (s + 1)) / splits);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) review_pool_kernel(SsdArgs a)
{
    const int cell = blockIdx.x, b = blockIdx.z / a.pool_splits, sp = blockIdx.z % a.pool_splits;
    const int CX = a.nh * a.P, CD = a.nh, CB = a.G * a.Ns, CH = CX + CD + CB;
    const int ch = blockIdx.y * blockDim.x + threadIdx.x;
    if (ch >= CH) return;
    const int hw = a.Hp * a.Wp;
    const int tp = cell / hw, r = cell - tp * hw, hp = r / a.Wp, wp = r - hp * a.Wp;
    const T *x = static_cast<const T *>(a.x);
    const T *Bm = static_cast<const T *>(a.B);
    int lo, hi;
    split_range(a.pt * a.ph * a.pw, a.pool_splits, sp, lo, hi);
    float sum = 0.f;
    for (int q = lo; q < hi; ++q) {
        const int i = q / (a.ph * a.pw), rr = q - i * (a.ph * a.pw), j = rr / a.pw, k = rr - j * a.pw;
        const int g = ((tp * a.pt + i) * a.H + hp * a.ph + j) * a.W + wp * a.pw + k;
        const size_t tok = tok_index(a, b, g);
        if (ch < CX)
            sum += ld(x + tok * CX + ch);
        else if (ch < CX + CD)
            sum += a.dt[tok * CD + (ch - CX)];
        else
            sum += ld(Bm + tok * CB + (ch - CX - CD));
    }
    a.pooled[(((size_t)b * a.pool_splits + sp) * a.Np + cell) * CH + ch] = sum;
}

// ---------------------------------------------------------------------------
// review_pool, vectorised for bf16 storage: each thread sums one 16-byte vector
// (8 channels of x or B) or one float4 of dt over its part of the cell's box.
// The block first lists the grid index of every token of that part in shared
// memory (kPoolTokens at a time), so the summing loop has no index arithmetic
// beyond one multiply-add per token, and it keeps eight 16-byte loads in
// flight per thread.
// grid: (Np, ceil(vectors / 256), batch * pool_splits); needs nh*P % 8 == 0,
// G*Ns % 8 == 0, nh % 4 == 0 and a 16-byte aligned dt.
// ---------------------------------------------------------------------------
constexpr int kPoolTokens = 1024;
constexpr int kPoolInFlight = 8;

__global__ void __launch_bounds__(kThreads) review_pool_vec_kernel(SsdArgs a)
{
    __shared__ int s_tok[kPoolTokens];
    const int cell = blockIdx.x, b = blockIdx.z / a.pool_splits, sp = blockIdx.z % a.pool_splits;
    const int CX = a.nh * a.P, CD = a.nh, CB = a.G * a.Ns, CH = CX + CD + CB;
    const int VX = CX / 8, VB = CB / 8, VD = CD / 4;
    const int v = blockIdx.y * blockDim.x + threadIdx.x;
    const bool active = v < VX + VB + VD;
    const int hw = a.Hp * a.Wp;
    const int tp = cell / hw, r = cell - tp * hw, hp = r / a.Wp, wp = r - hp * a.Wp;
    const int kind = v < VX ? 0 : (v < VX + VB ? 1 : 2);
    // this thread's 16 bytes of token 0 of batch element b, and the token stride
    const char *base;
    size_t stride;
    if (kind == 0) {
        base = reinterpret_cast<const char *>(static_cast<const __nv_bfloat16 *>(a.x) + (size_t)b * a.N * CX + v * 8);
        stride = (size_t)CX * 2;
    } else if (kind == 1) {
        base = reinterpret_cast<const char *>(static_cast<const __nv_bfloat16 *>(a.B) + (size_t)b * a.N * CB +
                                              (v - VX) * 8);
        stride = (size_t)CB * 2;
    } else {
        base = reinterpret_cast<const char *>(a.dt + (size_t)b * a.N * CD + (v - VX - VB) * 4);
        stride = (size_t)CD * 4;
    }
    int lo, hi;
    split_range(a.pt * a.ph * a.pw, a.pool_splits, sp, lo, hi);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int t0 = lo; t0 < hi; t0 += kPoolTokens) {
        const int cnt = min(kPoolTokens, hi - t0);
        __syncthreads();  // the previous list is no longer read
        for (int q = threadIdx.x; q < cnt; q += blockDim.x) {
            const int i = t0 + q;
            const int it = i / (a.ph * a.pw), rr = i - it * (a.ph * a.pw), ih = rr / a.pw, iw = rr - ih * a.pw;
            s_tok[q] = ((tp * a.pt + it) * a.H + hp * a.ph + ih) * a.W + wp * a.pw + iw;
        }
        __syncthreads();
        if (!active) continue;
        for (int q0 = 0; q0 < cnt; q0 += kPoolInFlight) {
            uint4 w[kPoolInFlight];
#pragma unroll
            for (int u = 0; u < kPoolInFlight; ++u)
                w[u] = q0 + u < cnt ? *reinterpret_cast<const uint4 *>(base + (size_t)s_tok[q0 + u] * stride)
                                    : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < kPoolInFlight; ++u) {
                if (kind == 2) {
                    acc[0] += __uint_as_float(w[u].x);
                    acc[1] += __uint_as_float(w[u].y);
                    acc[2] += __uint_as_float(w[u].z);
                    acc[3] += __uint_as_float(w[u].w);
                } else {
                    // bf16 pair -> two floats: the low half shifted up, the high half masked
                    acc[0] += __uint_as_float(w[u].x << 16);
                    acc[1] += __uint_as_float(w[u].x & 0xffff0000u);
                    acc[2] += __uint_as_float(w[u].y << 16);
                    acc[3] += __uint_as_float(w[u].y & 0xffff0000u);
                    acc[4] += __uint_as_float(w[u].z << 16);
                    acc[5] += __uint_as_float(w[u].z & 0xffff0000u);
                    acc[6] += __uint_as_float(w[u].w << 16);
                    acc[7] += __uint_as_float(w[u].w & 0xffff0000u);
                }
            }
        }
    }
    if (!active) return;
    float *dst = a.pooled + (((size_t)b * a.pool_splits + sp) * a.Np + cell) * CH;
    if (kind == 0) {
        dst += v * 8;
    } else if (kind == 1) {
        dst += CX + CD + (v - VX) * 8;
    } else {
        dst += CX + (v - VX - VB) * 4;
    }
    const int n = kind == 2 ? 4 : 8;
#pragma unroll
    for (int e = 0; e < 8; ++e)
        if (e < n) dst[e] = acc[e];
}

// ---------------------------------------------------------------------------
// review_scan: h_init[b][h] = state after scanning [R, flip(R)] from zero,
// R = pooled grid in scan order. The P rows of the state evolve independently,
// so RS CTAs split them. The review tokens are staged RT positions at a time
// (their grid cells listed first, so each value is one gather of the partial
// box sums). grid: (nh, batch, RS)
// ---------------------------------------------------------------------------
template <int P, int NS, int RS>
__global__ void __launch_bounds__(kThreads) review_scan_kernel(SsdArgs a)
{
    constexpr int PR = P / RS;  // state rows of this CTA
    constexpr int PN = PR * NS;
    // thread t owns E consecutive elements t*E .. of the PR x NS block (one state
    // row, adjacent columns): four per thread when they fill the CTA, else one
    constexpr int E = (NS % 4 == 0 && PN >= 4 * kThreads) ? 4 : 1;
    constexpr int NE = (PN + E * kThreads - 1) / (E * kThreads);  // element groups per thread
    constexpr int W = (PR + NS + 1 + 3) & ~3;                     // x rows | B | decay, padded to 16 bytes
    constexpr int RT = W * 128 * 4 <= 44 * 1024 ? 128 : 32;       // positions per staged tile
    __shared__ __align__(16) float vals[RT][W];
    __shared__ int cells[RT];
    const int h = blockIdx.x, b = blockIdx.y, p0 = blockIdx.z * PR;
    const int grp = h / (a.nh / a.G);
    const int CX = a.nh * a.P, CD = a.nh, CH = CX + CD + a.G * a.Ns;
    const float Ah = a.A[h];
    const int L = 2 * a.Np;
    const float inv_box = 1.f / (float)(a.pt * a.ph * a.pw);
    constexpr int WV = PR + NS + 1;  // staged values per position
    float s[NE][E];
#pragma unroll
    for (int u = 0; u < NE; ++u)
#pragma unroll
        for (int e = 0; e < E; ++e) s[u][e] = 0.f;
    for (int base = 0; base < L; base += RT) {
        __syncthreads();  // the previous tile is consumed
        for (int k = threadIdx.x; k < RT; k += blockDim.x) {
            const int pos = base + k;
            const int r = pos < a.Np ? pos : L - 1 - pos;  // [R, flip(R)]
            cells[k] = pos < L ? rms_grid_offset(r, a.Tp, a.Hp, a.Wp, a.mode) : 0;
        }
        __syncthreads();
        const int kmax = min(RT, L - base);
        // eight gathers in flight per thread
        constexpr int kU = 8;
        for (int i0 = threadIdx.x; i0 < kmax * WV; i0 += kU * blockDim.x) {
            const float *src[kU];
            float v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int idx = min(i0 + u * (int)blockDim.x, kmax * WV - 1);
                const int k = idx / WV, c = idx - k * WV;
                const int col = c < PR ? h * P + p0 + c : (c < PR + NS ? CX + CD + grp * NS + (c - PR) : CX + h);
                src[u] = a.pooled + ((size_t)b * a.pool_splits * a.Np + cells[k]) * CH + col;
                v[u] = 0.f;
            }
            for (int sp = 0; sp < a.pool_splits; ++sp)
#pragma unroll
                for (int u = 0; u < kU; ++u) v[u] += src[u][(size_t)sp * a.Np * CH];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int idx = i0 + u * (int)blockDim.x;
                if (idx < kmax * WV) {
                    const int k = idx / WV, c = idx - k * WV;
                    vals[k][c] = v[u] * inv_box;
                }
            }
        }
        __syncthreads();
        // per position: the decay exp(dt A) (kept in the dt slot) and dt x
        for (int k = threadIdx.x; k < kmax; k += blockDim.x) {
            const float dk = vals[k][PR + NS];
#pragma unroll
            for (int p = 0; p < PR; ++p) vals[k][p] *= dk;
            vals[k][PR + NS] = expf(dk * Ah);
        }
        __syncthreads();
        for (int k = 0; k < kmax; ++k) {
            const float dec = vals[k][PR + NS];
#pragma unroll
            for (int u = 0; u < NE; ++u) {
                const int i0 = (threadIdx.x + u * kThreads) * E;
                if (i0 < PN) {
                    const int p = i0 / NS, n = i0 - p * NS;
                    const float xp = vals[k][p];
                    if (E == 4) {
                        const float4 bv = *reinterpret_cast<const float4 *>(&vals[k][PR + n]);
                        s[u][0] = fmaf(dec, s[u][0], xp * bv.x);
                        s[u][1] = fmaf(dec, s[u][1], xp * bv.y);
                        s[u][2] = fmaf(dec, s[u][2], xp * bv.z);
                        s[u][3] = fmaf(dec, s[u][3], xp * bv.w);
                    } else {
#pragma unroll
                        for (int e = 0; e < E; ++e) s[u][e] = fmaf(dec, s[u][e], xp * vals[k][PR + n + e]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < NE; ++u) {
        const int i0 = (threadIdx.x + u * kThreads) * E;
#pragma unroll
        for (int e = 0; e < E; ++e)
            if (i0 + e < PN) a.h_init[((size_t)b * a.nh + h) * (P * NS) + p0 * NS + i0 + e] = s[u][e];
    }
}

// ---------------------------------------------------------------------------
// review_hinit (P = Ns = 64): h_init without a sequential scan. Scanning the
// prefix [R, flip(R)] (2 Np positions) from zero leaves
//   h = sum_j exp(A * sum_{k>j} dt_k) * dt_j * x_j B_j^T,
// and cell r of R sits at positions r and 2 Np - 1 - r. With d_r the cell's
// pooled dt, P_r = sum_{r'<r} d_r' (the dt after position 2 Np - 1 - r) and
// D = sum_r d_r (so 2D - P_r - d_r is the dt after position r):
//   h = sum_r W_r x_r B_r^T,   W_r = d_r (exp(A P_r) + exp(A (2D - P_r - d_r))).
// CTA z takes the z-th of kHinitParts ranges of cells and writes its part of
// the sum to h_init part z; the state chain adds the parts. grid: (nh, batch,
// kHinitParts)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 3) review_hinit_kernel(SsdArgs a)
{
    constexpr int P = 64, NS = 64, RT = 64;  // RT: cells per staged tile
    constexpr int kDCap = 1024;              // pooled dt kept in shared memory up to this many cells
    constexpr int kLd = RT * 32 / kThreads;  // 16-byte loads per thread per tile
    __shared__ __align__(16) float xs[RT][P];
    __shared__ __align__(16) float bs[RT][NS];
    __shared__ float ws[RT];
    __shared__ float dsm[kDCap];
    __shared__ float red[2][kThreads / 32];
    const int h = blockIdx.x, b = blockIdx.y, part = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = h / (a.nh / a.G);
    const int CX = a.nh * P, CD = a.nh, CH = CX + CD + a.G * NS;
    const float Ah = a.A[h];
    const float inv_box = 1.f / (float)(a.pt * a.ph * a.pw);
    const float *pb = a.pooled + (size_t)b * a.pool_splits * a.Np * CH;
    const size_t split_stride = (size_t)a.Np * CH;
    const bool vec = (CH & 3) == 0, dcache = a.Np <= kDCap;
    int r0, r1;
    split_range(a.Np, kHinitParts, part, r0, r1);
    // pooled dt of the cell at position r of R (a box mean)
    auto dbar = [&](int r) {
        const float *src = pb + (size_t)rms_grid_offset(r, a.Tp, a.Hp, a.Wp, a.mode) * CH + CX + h;
        float d = 0.f;
        for (int sp = 0; sp < a.pool_splits; ++sp) d += src[sp * split_stride];
        return d * inv_box;
    };
    // the loads of one tile's x rows (this head) and B rows (this group): box sums, four
    // values a load, all of a thread's loads in flight at once
    const float *src[kLd];
    float4 v[kLd];
    auto tile_loads = [&](int t0, int cnt) {
#pragma unroll
        for (int j = 0; j < kLd; ++j) {
            const int i = tid + j * kThreads, k = min(i >> 5, cnt - 1), q = i & 31;
            src[j] = pb + (size_t)rms_grid_offset(t0 + k, a.Tp, a.Hp, a.Wp, a.mode) * CH +
                     (q < 16 ? h * P + 4 * q : CX + CD + grp * NS + 4 * (q - 16));
            v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int sp = 0; sp < a.pool_splits; ++sp) {
#pragma unroll
            for (int j = 0; j < kLd; ++j) {
                const float *s4 = src[j] + sp * split_stride;
                const float4 u = vec ? *reinterpret_cast<const float4 *>(s4) : make_float4(s4[0], s4[1], s4[2], s4[3]);
                v[j].x += u.x, v[j].y += u.y, v[j].z += u.z, v[j].w += u.w;
            }
        }
    };
    if (r0 < r1) tile_loads(r0, min(RT, r1 - r0));  // the first tile's rows load meanwhile
    // D, and P_r at the first cell of this part
    float dall = 0.f, dpre = 0.f;
    for (int r = tid; r < a.Np; r += kThreads) {
        const float d = dbar(r);
        if (dcache) dsm[r] = d;
        dall += d;
        if (r < r0) dpre += d;
    }
    dall = warp_sum(dall);
    dpre = warp_sum(dpre);
    if (lane == 0) {
        red[0][warp] = dall;
        red[1][warp] = dpre;
    }
    __syncthreads();
    float D2 = 0.f, carry = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        D2 += red[0][w];
        carry += red[1][w];
    }
    D2 *= 2.f;
    // thread: state rows 4 (t / 16) .. + 3, columns 4 (t % 16) .. + 3
    const int p4 = (tid >> 4) * 4, n4 = (tid & 15) * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int t0 = r0; t0 < r1; t0 += RT) {
        const int cnt = min(RT, r1 - t0);
        if (t0 != r0) {
            __syncthreads();  // the previous tile is consumed
            tile_loads(t0, cnt);
        }
#pragma unroll
        for (int j = 0; j < kLd; ++j) {
            const int i = tid + j * kThreads, k = i >> 5, q = i & 31;
            if (k < cnt) *reinterpret_cast<float4 *>(q < 16 ? &xs[k][4 * q] : &bs[k][4 * (q - 16)]) = v[j];
        }
        if (warp == 0) {
            // the tile's weights, two cells a lane, from an exclusive prefix of d over the tile;
            // 1/box twice turns the x and B sums into means
            const int k0 = 2 * lane;
            float d0 = 0.f, d1 = 0.f;
            if (k0 < cnt) d0 = dcache ? dsm[t0 + k0] : dbar(t0 + k0);
            if (k0 + 1 < cnt) d1 = dcache ? dsm[t0 + k0 + 1] : dbar(t0 + k0 + 1);
            const float incl = warp_inclusive_scan(d0 + d1);
            const float p0 = carry + incl - (d0 + d1), p1 = p0 + d0;
            const float sc = inv_box * inv_box;
            if (k0 < cnt) ws[k0] = d0 * (expf(Ah * p0) + expf(Ah * (D2 - p0 - d0))) * sc;
            if (k0 + 1 < cnt) ws[k0 + 1] = d1 * (expf(Ah * p1) + expf(Ah * (D2 - p1 - d1))) * sc;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncthreads();
        for (int k = 0; k < cnt; ++k) {
            const float w = ws[k];
            const float4 xv = *reinterpret_cast<const float4 *>(&xs[k][p4]);
            const float4 bv = *reinterpret_cast<const float4 *>(&bs[k][n4]);
            const float xw[4] = {xv.x * w, xv.y * w, xv.z * w, xv.w * w};
            const float2 b01 = make_float2(bv.x, bv.y), b23 = make_float2(bv.z, bv.w);
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // packed fp32 pairs
                const float2 x2 = make_float2(xw[i], xw[i]);
                const float2 a01 = tc::fma_f32x2(x2, b01, make_float2(acc[i][0], acc[i][1]));
                const float2 a23 = tc::fma_f32x2(x2, b23, make_float2(acc[i][2], acc[i][3]));
                acc[i][0] = a01.x, acc[i][1] = a01.y, acc[i][2] = a23.x, acc[i][3] = a23.y;
            }
        }
    }
    float *dst = a.h_init + (((size_t)part * a.batch + b) * a.nh + h) * (P * NS) + p4 * NS + n4;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float4 *>(dst + i * NS) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
}

// ---------------------------------------------------------------------------
// chunk_state: chunk-local states from a zero start
//   forward : sum_j exp(cum_end - cum_j) dt_j x_j B_j^T
//   flipped : sum_j exp(excl_j) dt_j x_j B_j^T
//   alpha   : exp(cum_end)
// grid: (nchunks, nh, batch)
// ---------------------------------------------------------------------------
template <typename T, int P, int NS>
__global__ void __launch_bounds__(kThreads) chunk_state_kernel(SsdArgs a)
{
    constexpr int PN = P * NS;
    constexpr int E = (PN + kThreads - 1) / kThreads;
    __shared__ float cum[kMaxStateChunk];
    __shared__ float dts[kMaxStateChunk];
    __shared__ int goff[kMaxStateChunk];
    __shared__ float xs[kTile][P];
    __shared__ float bs[kTile][NS];
    __shared__ float wf[kTile], wb[kTile];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int n0 = c * a.Q, len = min(a.Q, a.N - n0);
    const int grp = h / (a.nh / a.G);
    const float Ah = a.A[h];
    const T *x = static_cast<const T *>(a.x);
    const T *Bm = static_cast<const T *>(a.B);
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
        const int g = rms_grid_offset(n0 + i, a.T, a.H, a.W, a.mode);
        goff[i] = g;
        const float d = a.dt[tok_index(a, b, g) * a.nh + h];
        dts[i] = d;
        cum[i] = d * Ah;
    }
    block_inclusive_scan(cum, len);
    const float cend = cum[len - 1];
    float sf[E], sb[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sf[e] = sb[e] = 0.f;
    for (int base = 0; base < len; base += kTile) {
        const int kmax = min(kTile, len - base);
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTile * (P + NS); idx += blockDim.x) {
            const int k = idx / (P + NS), col = idx - k * (P + NS);
            if (k >= kmax) continue;
            const size_t tok = tok_index(a, b, goff[base + k]);
            if (col < P)
                xs[k][col] = ld(x + (tok * a.nh + h) * P + col);
            else
                bs[k][col - P] = ld(Bm + (tok * a.G + grp) * NS + (col - P));
        }
        if (threadIdx.x < kmax) {
            const int i = base + threadIdx.x;
            wf[threadIdx.x] = expf(cend - cum[i]) * dts[i];
            wb[threadIdx.x] = expf(cum[i] - dts[i] * Ah) * dts[i];
        }
        __syncthreads();
        for (int k = 0; k < kmax; ++k) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int idx = threadIdx.x + e * kThreads;
                if (idx < PN) {
                    const int p = idx / NS, n = idx - p * NS;
                    const float v = xs[k][p] * bs[k][n];
                    sf[e] += wf[k] * v;
                    sb[e] += wb[k] * v;
                }
            }
        }
    }
    const size_t base_out = (((size_t)b * a.nh + h) * a.nchunks + c) * PN;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int idx = threadIdx.x + e * kThreads;
        if (idx < PN) {
            a.states_f[base_out + idx] = sf[e];
            a.states_b[base_out + idx] = sb[e];
        }
    }
    if (threadIdx.x == 0) a.alpha[((size_t)b * a.nh + h) * a.nchunks + c] = expf(cend);
}

// ---------------------------------------------------------------------------
// state_pass: replace every chunk-local state by the state entering that
// chunk (forward: from the left; flipped: from the right). Both start from
// h_init with review tokens, else from zero. grid: (nh, batch, 2)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) state_pass_kernel(SsdArgs a)
{
    const int h = blockIdx.x, b = blockIdx.y, dir = blockIdx.z;
    if (!(a.dirs & (1 << dir))) return;
    const int PN = a.P * a.Ns, nc = a.nchunks;
    float *S = (dir == 0 ? a.states_f : a.states_b) + ((size_t)b * a.nh + h) * nc * PN;
    const float *al = a.alpha + ((size_t)b * a.nh + h) * nc;
    for (int idx = threadIdx.x; idx < PN; idx += blockDim.x) {
        float Hv = a.review ? a.h_init[((size_t)b * a.nh + h) * PN + idx] : 0.f;
        if (dir == 0) {
            float nxt = S[idx];
            for (int c = 0; c < nc; ++c) {
                const float cur = nxt;
                if (c + 1 < nc) nxt = S[(size_t)(c + 1) * PN + idx];
                S[(size_t)c * PN + idx] = Hv;
                Hv = al[c] * Hv + cur;
            }
        } else {
            float nxt = S[(size_t)(nc - 1) * PN + idx];
            for (int c = nc - 1; c >= 0; --c) {
                const float cur = nxt;
                if (c > 0) nxt = S[(size_t)(c - 1) * PN + idx];
                S[(size_t)c * PN + idx] = Hv;
                Hv = al[c] * Hv + cur;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// chunk_out: one thread per token of the chunk.
// grid: (nchunks, nh, batch); block: 256; dynamic shared memory:
//   bs[Q][NS] xs[Q][P] Hf[P][NS] Hb[P][NS] cum[Q] dts[Q] goff[Q]
// ---------------------------------------------------------------------------
template <typename T, int P, int NS>
__global__ void __launch_bounds__(kThreads) chunk_out_kernel(SsdArgs a)
{
    extern __shared__ float smem[];
    const int Q = a.Q;
    float *bs = smem;
    float *xs = bs + (size_t)Q * NS;
    float *Hf = xs + (size_t)Q * P;
    float *Hb = Hf + P * NS;
    float *cum = Hb + P * NS;
    float *dts = cum + Q;
    int *goff = reinterpret_cast<int *>(dts + Q);

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int n0 = c * Q, len = min(Q, a.N - n0);
    const int grp = h / (a.nh / a.G);
    const float Ah = a.A[h], Dh = a.D[h];
    const bool fwd = a.dirs & 1, bwd = a.dirs & 2;
    const T *x = static_cast<const T *>(a.x);
    const T *Bm = static_cast<const T *>(a.B);
    const T *Cm = static_cast<const T *>(a.C);
    T *out = static_cast<T *>(a.out);

    for (int i = threadIdx.x; i < len; i += blockDim.x) {
        const int g = rms_grid_offset(n0 + i, a.T, a.H, a.W, a.mode);
        goff[i] = g;
        const float d = a.dt[tok_index(a, b, g) * a.nh + h];
        dts[i] = d;
        cum[i] = d * Ah;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < len * (P + NS); idx += blockDim.x) {
        const int i = idx / (P + NS), col = idx - i * (P + NS);
        const size_t tok = tok_index(a, b, goff[i]);
        if (col < P)
            xs[i * P + col] = ld(x + (tok * a.nh + h) * P + col);
        else
            bs[i * NS + (col - P)] = ld(Bm + (tok * a.G + grp) * NS + (col - P));
    }
    const size_t sbase = (((size_t)b * a.nh + h) * a.nchunks + c) * (P * NS);
    for (int idx = threadIdx.x; idx < P * NS; idx += blockDim.x) {
        Hf[idx] = fwd ? a.states_f[sbase + idx] : 0.f;
        Hb[idx] = bwd ? a.states_b[sbase + idx] : 0.f;
    }
    block_inclusive_scan(cum, len);

    const int i = threadIdx.x;
    if (i >= len) return;
    const size_t tok = tok_index(a, b, goff[i]);
    float ci[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) ci[n] = ld(Cm + (tok * a.G + grp) * NS + n);
    float y[P];
#pragma unroll
    for (int p = 0; p < P; ++p) y[p] = 0.f;
    const float cum_i = cum[i];
    const float excl_i = cum_i - dts[i] * Ah;
    const float cend = cum[len - 1];
    for (int j = 0; j < len; ++j) {
        float w = 0.f;
        if (fwd && j <= i) w += expf(cum_i - cum[j]);
        if (bwd && j >= i) w += expf((cum[j] - dts[j] * Ah) - excl_i);
        if (w == 0.f) continue;
        float s = 0.f;
#pragma unroll
        for (int n = 0; n < NS; ++n) s += ci[n] * bs[j * NS + n];
        w *= s * dts[j];
#pragma unroll
        for (int p = 0; p < P; ++p) y[p] += w * xs[j * P + p];
    }
    const float rf = fwd ? expf(cum_i) : 0.f;
    const float rb = bwd ? expf(cend - excl_i) : 0.f;
    const float dx = (float)((int)fwd + (int)bwd) * Dh;
#pragma unroll
    for (int p = 0; p < P; ++p) {
        float zf = 0.f, zb = 0.f;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            zf += ci[n] * Hf[p * NS + n];
            zb += ci[n] * Hb[p * NS + n];
        }
        y[p] += rf * zf + rb * zb + dx * xs[i * P + p];
    }
    T *o = out + (tok * a.nh + h) * P;
#pragma unroll
    for (int p = 0; p < P; ++p) st(o + p, y[p]);
}

// review prefix, chunk-local states and the state chain: everything before
// the chunk outputs
template <typename T, int P, int NS>
cudaError_t run_prepass(const SsdArgs &a, cudaStream_t s)
{
    if (a.review) {
        const int CH = a.nh * a.P + a.nh + a.G * a.Ns;
        {
            Phase ph(MATE_PHASE_REVIEW_POOL, s);
            review_pool_kernel<T><<<dim3(a.Np, (CH + kThreads - 1) / kThreads, a.batch * a.pool_splits), kThreads, 0, s>>>(a);
        }
        {
            Phase ph(MATE_PHASE_REVIEW_SCAN, s);
            constexpr int RS = P >= 32 ? P / 16 : 1;
            review_scan_kernel<P, NS, RS><<<dim3(a.nh, a.batch, RS), kThreads, 0, s>>>(a);
        }
    }
    {
        Phase ph(MATE_PHASE_CHUNK_STATE, s);
        chunk_state_kernel<T, P, NS><<<dim3(a.nchunks, a.nh, a.batch), kThreads, 0, s>>>(a);
    }
    {
        Phase ph(MATE_PHASE_STATE_PASS, s);
        state_pass_kernel<<<dim3(a.nh, a.batch, 2), kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

template <typename T, int P, int NS>
cudaError_t run(const SsdArgs &a, cudaStream_t s)
{
    const size_t smem = ((size_t)a.Q * (P + NS) + 2 * P * NS + 3 * (size_t)a.Q) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(chunk_out_kernel<T, P, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    e = run_prepass<T, P, NS>(a, s);
    if (e != cudaSuccess) return e;
    {
        Phase ph(MATE_PHASE_CHUNK_OUT, s);
        chunk_out_kernel<T, P, NS><<<dim3(a.nchunks, a.nh, a.batch), kThreads, smem, s>>>(a);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_dims(const SsdArgs &a, cudaStream_t s)
{
#define MATE_CASE(PP, NN) \
    if (a.P == PP && a.Ns == NN) return run<T, PP, NN>(a, s);
    MATE_CASE(16, 16) MATE_CASE(16, 32) MATE_CASE(16, 64)
    MATE_CASE(32, 16) MATE_CASE(32, 32) MATE_CASE(32, 64)
    MATE_CASE(64, 16) MATE_CASE(64, 32) MATE_CASE(64, 64)
#undef MATE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_ssd_generic(const SsdArgs &a, cudaStream_t s)
{
    // fp32 storage only: bf16 calls run on the tensor-core kernels or are refused
    return a.bf16 ? cudaErrorInvalidValue : dispatch_dims<float>(a, s);
}

cudaError_t launch_review_bf16_64(const SsdArgs &a, cudaStream_t s)
{
    const cudaError_t e = launch_review_pool_bf16_64(a, s);
    return e != cudaSuccess ? e : launch_review_scan_bf16_64(a, s);
}

cudaError_t launch_review_pool_bf16_64(const SsdArgs &a, cudaStream_t s)
{
    const int CH = a.nh * a.P + a.nh + a.G * a.Ns;
    const bool vec = (a.nh * a.P) % 8 == 0 && (a.G * a.Ns) % 8 == 0 && a.nh % 4 == 0 &&
                     reinterpret_cast<uintptr_t>(a.dt) % 16 == 0;  // dt is read as float4
    {
        Phase ph(MATE_PHASE_REVIEW_POOL, s);
        if (vec) {
            const int nv = a.nh * a.P / 8 + a.G * a.Ns / 8 + a.nh / 4;
            review_pool_vec_kernel<<<dim3(a.Np, (nv + kThreads - 1) / kThreads, a.batch * a.pool_splits), kThreads, 0,
                                     s>>>(a);
        } else {
            review_pool_kernel<__nv_bfloat16>
                <<<dim3(a.Np, (CH + kThreads - 1) / kThreads, a.batch * a.pool_splits), kThreads, 0, s>>>(a);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_review_scan_bf16_64(const SsdArgs &a, cudaStream_t s)
{
    {
        Phase ph(MATE_PHASE_REVIEW_SCAN, s);
        review_hinit_kernel<<<dim3(a.nh, a.batch, kHinitParts), kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace mate
