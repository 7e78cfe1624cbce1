// Chunk outputs of the bidirectional SSD scan on the 5th-generation tensor
// cores (tcgen05 + TMEM) for bf16 storage, head dim 64, d_state 64.
//
// Method (paper review "LinGen ...", section 三, MA-Branch items 1-2): per
// head, the Mamba2 recurrence s_n = exp(dt_n A) s_{n-1} + dt_n x_n B_n^T,
// y_n = s_n C_n + D x_n, over the Rotary-Major-Scan sequence and over its
// flip, flipped back and added.
//
// One CTA per (head, chunk of L = 128*K tokens, batch element); the states
// entering the chunk from the left (forward scan) and from the right (flipped
// scan) come from the chunk-state chain. Inside the chunk, K sub-chunks of
// 128 tokens:
//   phase 1  for each sub-chunk, both sub-chunk-local states in one MMA:
//            [ (w_f x)^T ; (w_b x)^T ] (128 x 128 tokens) . B (128 tokens x 64)
//            with w_f[j] = exp(c_end - c_j) dt_j and w_b[j] = exp(e_j) dt_j
//            (c: inclusive, e: exclusive cumulative sum of A dt inside the
//            sub-chunk), rows 0-63 forward, rows 64-127 flipped, kept in TMEM.
//   phase 2  chain them in TMEM: each lane owns one state row; the forward
//            lanes walk the sub-chunks left to right, the flipped lanes right
//            to left, replacing every local state by the state entering it.
//   phase 3  for each sub-chunk, S = C B^T (128 x 128) into TMEM; thread i
//            turns row i of S into row i of
//               A = [ M | R_f C | R_b C ]   (128 x 256, bf16)
//            with M_ij = S_ij dt_j (exp(c_i - c_j) [j <= i] + exp(e_j - e_i) [j >= i]),
//            R_f[i] = exp(c_i), R_b[i] = exp(c_end - e_i); then one accumulating
//            MMA chain computes A . [ x ; h_f^T ; h_b^T ] (256 x 64), and the
//            epilogue adds 2 D x and stores the row to its grid position.
// The exponentials of M are factored around the sub-chunk midpoint,
// exp(c_i - c_j) = exp(c_i - r) exp(r - c_j), so a row costs two exps per
// element pair only when the sub-chunk's decay range is too wide for fp32
// (then every element is exponentiated exactly).
// The RMS order enters only through the gather addresses: row j of a
// sub-chunk is the grid token of scan position n = chunk start + j.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace mate {

namespace {

constexpr int kThreads = 128;
constexpr int kSub = 128;        // tokens per sub-chunk
constexpr int kMaxSubs = 4;      // sub-chunks per chunk held in TMEM
constexpr uint32_t kTile = 16384;

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffX = 0;                 // 2 buffers x 16 KB
constexpr uint32_t kOffB = 2 * kTile;         // 2 buffers
constexpr uint32_t kOffC = 4 * kTile;         // 2 buffers
constexpr uint32_t kOffA = 6 * kTile;         // 4 tiles: phase 1 U_f, U_b; phase 3 M0, M1, Cf, Cb
constexpr uint32_t kOffH = 10 * kTile;        // h_f (8 KB) then h_b (8 KB)
constexpr uint32_t kOffF = 11 * kTile;        // fp32 / int arrays
constexpr int kMaxChunk = kSub * kMaxSubs;
// arrays after kOffF: dt[512], cum[512] (inclusive, sub-chunk local), goff[512],
// gf[128], gb[128], misc
constexpr uint32_t kOffDt = kOffF;
constexpr uint32_t kOffCum = kOffDt + kMaxChunk * 4;
constexpr uint32_t kOffGoff = kOffCum + kMaxChunk * 4;
constexpr uint32_t kOffGf = kOffGoff + kMaxChunk * 4;
constexpr uint32_t kOffGb = kOffGf + kSub * 4;
constexpr uint32_t kOffRed = kOffGb + kSub * 4;     // 8 floats of block reductions
constexpr uint32_t kOffBar = kOffRed + 64;
constexpr uint32_t kSmemUsed = kOffBar + 64;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;

// TMEM columns
constexpr uint32_t kColS = kMaxSubs * 64;   // S (128 cols) after the K state slots
constexpr uint32_t kColAcc = kColS + 128;   // output accumulator (64 cols)
constexpr uint32_t kTmemCols = 512;

constexpr float kFactorLimit = 80.f;        // |exponent| bound for the factored exps

struct Smem {
    uint8_t *base;
    __device__ uint8_t *X(int buf) const { return base + kOffX + buf * kTile; }
    __device__ uint8_t *B(int buf) const { return base + kOffB + buf * kTile; }
    __device__ uint8_t *C(int buf) const { return base + kOffC + buf * kTile; }
    __device__ uint8_t *A(int t) const { return base + kOffA + t * kTile; }
    __device__ uint8_t *Hf() const { return base + kOffH; }
    __device__ uint8_t *Hb() const { return base + kOffH + 8192; }
    __device__ float *dt() const { return reinterpret_cast<float *>(base + kOffDt); }
    __device__ float *cum() const { return reinterpret_cast<float *>(base + kOffCum); }
    __device__ int *goff() const { return reinterpret_cast<int *>(base + kOffGoff); }
    __device__ float *gf() const { return reinterpret_cast<float *>(base + kOffGf); }
    __device__ float *gb() const { return reinterpret_cast<float *>(base + kOffGb); }
    __device__ float *red() const { return reinterpret_cast<float *>(base + kOffRed); }
    __device__ uint64_t *bar() const { return reinterpret_cast<uint64_t *>(base + kOffBar); }
    __device__ uint32_t *tmem_slot() const { return reinterpret_cast<uint32_t *>(base + kOffBar + 8); }
    __device__ int *abort_flag() const { return reinterpret_cast<int *>(base + kOffBar + 12); }
};

// Gather the 128 token rows of sub-chunk `sub` into swizzled tiles (x: 64 head
// dims of head h; B and C: 64 state dims of the head's group). Rows past the
// sequence end are zero.
__device__ __forceinline__ void load_rows(const SsdArgs &a, const Smem &sm, int b, int h, int grp, int n0, int len,
                                          int sub, int buf, bool withC)
{
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a.x);
    const __nv_bfloat16 *Bm = static_cast<const __nv_bfloat16 *>(a.B);
    const __nv_bfloat16 *Cm = static_cast<const __nv_bfloat16 *>(a.C);
    const int ntiles = withC ? 3 : 2;
    for (int idx = threadIdx.x; idx < ntiles * kSub * 8; idx += kThreads) {
        const int tile = idx / (kSub * 8);
        const int r = (idx / 8) % kSub, c = idx % 8;
        const int n = sub * kSub + r;  // position inside the chunk
        uint8_t *dst = (tile == 0 ? sm.X(buf) : tile == 1 ? sm.B(buf) : sm.C(buf)) + tc::sw128(r, c);
        if (n < len) {
            const size_t tok = (size_t)b * a.N + sm.goff()[n];
            const __nv_bfloat16 *src = tile == 0 ? x + (tok * a.nh + h) * 64 + c * 8
                                                 : (tile == 1 ? Bm : Cm) + (tok * a.G + grp) * 64 + c * 8;
            tc::cp_async16(dst, src);
        } else {
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
        }
    }
    tc::cp_async_commit();
}

__device__ __forceinline__ void wait_loads(bool newer_pending)
{
    if (newer_pending)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
    else
        asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// 8 bf16 of a swizzled row -> floats
__device__ __forceinline__ void row_chunk(const uint8_t *tile, int r, int c, float (&v)[8])
{
    const uint4 u = *reinterpret_cast<const uint4 *>(tile + tc::sw128(r, c));
    float2 f;
    f = tc::unpack_bf16(u.x); v[0] = f.x; v[1] = f.y;
    f = tc::unpack_bf16(u.y); v[2] = f.x; v[3] = f.y;
    f = tc::unpack_bf16(u.z); v[4] = f.x; v[5] = f.y;
    f = tc::unpack_bf16(u.w); v[6] = f.x; v[7] = f.y;
}

__device__ __forceinline__ void put_chunk(uint8_t *tile, int r, int c, const float (&v)[8])
{
    uint4 u;
    u.x = tc::pack_bf16(v[0], v[1]);
    u.y = tc::pack_bf16(v[2], v[3]);
    u.z = tc::pack_bf16(v[4], v[5]);
    u.w = tc::pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + tc::sw128(r, c)) = u;
}

__device__ __forceinline__ float block_max128(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

__global__ void __launch_bounds__(kThreads, 1) ssd_chunk_out_tc_kernel(SsdArgs a, int nsub)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    Smem sm{smem_raw + ((1024u - (raw & 1023u)) & 1023u)};
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.x, c = blockIdx.y, b = blockIdx.z;
    const int L = nsub * kSub;
    const int n0 = c * L, len = min(L, a.N - n0);
    const int grp = h / (a.nh / a.G);
    const float Ah = a.A[h], Dh = a.D[h];
    uint64_t *bar = sm.bar();
    int *abort_flag = sm.abort_flag();
    uint32_t mma_phase = 0;

    if (warp == 0) tc::tmem_alloc(sm.tmem_slot(), kTmemCols);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    // scan positions -> grid offsets, dt, sub-chunk-local inclusive cumsum of A dt
    for (int n = tid; n < L; n += kThreads) {
        float d = 0.f;
        int g = 0;
        if (n < len) {
            g = rms_grid_offset(n0 + n, a.T, a.H, a.W, a.mode);
            d = a.dt[((size_t)b * a.N + g) * a.nh + h];
        }
        sm.goff()[n] = g;
        sm.dt()[n] = d;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot();

    // sub-chunk-local inclusive cumsums: warp w scans sub-chunk w (nsub <= 4)
    if (warp < nsub) {
        float carry = 0.f;
        for (int base = 0; base < kSub; base += 32) {
            const int n = warp * kSub + base + (tid & 31);
            float v = warp_inclusive_scan(sm.dt()[n] * Ah) + carry;
            sm.cum()[n] = v;
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();

    auto mma_wait = [&]() -> bool {
        const bool ok = tc::mbar_wait(bar, mma_phase & 1u, a.err);
        ++mma_phase;
        if (!ok) atomicExch(abort_flag, 1);
        __syncthreads();
        if (*abort_flag) {
            tc::mbar_wait(bar, (mma_phase - 1) & 1u, nullptr);
            return false;
        }
        tc::tc_fence_after();
        return true;
    };

    // ---------------- phase 1: sub-chunk-local states -> TMEM -------------------
    load_rows(a, sm, b, h, grp, n0, len, 0, 0, false);
    for (int k = 0; k < nsub; ++k) {
        const int buf = k & 1;
        if (k + 1 < nsub) load_rows(a, sm, b, h, grp, n0, len, k + 1, buf ^ 1, false);
        wait_loads(k + 1 < nsub);
        __syncthreads();
        {
            const int j = tid, n = k * kSub + j;
            const float cj = sm.cum()[n], dj = sm.dt()[n];
            const float cend = sm.cum()[k * kSub + kSub - 1];
            const float wf = __expf(cend - cj) * dj;
            const float wb = __expf(cj - dj * Ah) * dj;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float v[8], uf[8], ub[8];
                row_chunk(sm.X(buf), j, ch, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    uf[e] = wf * v[e];
                    ub[e] = wb * v[e];
                }
                put_chunk(sm.A(0), j, ch, uf);
                put_chunk(sm.A(1), j, ch, ub);
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t idesc = tc::idesc_bf16(128, 64, 1, 1);
            const uint32_t a0 = tc::smem_u32(sm.A(0)), b0 = tc::smem_u32(sm.B(buf));
#pragma unroll
            for (int s = 0; s < 8; ++s)
                tc::mma_bf16(tmem + k * 64, tc::sdesc_sw128(a0 + s * 2048, kTile, 1024),
                             tc::sdesc_sw128(b0 + s * 2048, kTile, 1024), idesc, s > 0);
            tc::mma_commit(bar);
        }
        if (!mma_wait()) goto cleanup;
    }

    // ---------------- phase 2: chain the sub-chunk states in TMEM ----------------
    {
        const bool fwd = warp < 2;
        const int p = fwd ? tid : tid - 64;
        const float *Hin = (fwd ? a.states_f : a.states_b) + ((((size_t)b * a.nh + h) * a.nchunks + c) * 64 + p) * 64;
        float hv[2][32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            hv[0][q] = Hin[q];
            hv[1][q] = Hin[32 + q];
        }
        const uint32_t lane_base = (uint32_t)(warp * 32);
        for (int it = 0; it < nsub; ++it) {
            const int k = fwd ? it : nsub - 1 - it;
            const float alpha = __expf(sm.cum()[k * kSub + kSub - 1]);
            float t0[32], t1[32];
            tc::tmem_ld32(tc::tmem_addr(tmem, lane_base, k * 64), t0);
            tc::tmem_ld32(tc::tmem_addr(tmem, lane_base, k * 64 + 32), t1);
            tc::tmem_wait_ld();
            tc::tmem_st32(tc::tmem_addr(tmem, lane_base, k * 64), hv[0]);
            tc::tmem_st32(tc::tmem_addr(tmem, lane_base, k * 64 + 32), hv[1]);
            tc::tmem_wait_st();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                hv[0][q] = fmaf(alpha, hv[0][q], t0[q]);
                hv[1][q] = fmaf(alpha, hv[1][q], t1[q]);
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    // ---------------- phase 3: outputs ------------------------------------------
    load_rows(a, sm, b, h, grp, n0, len, 0, 0, true);
    for (int k = 0; k < nsub; ++k) {
        const int buf = k & 1;
        if (k + 1 < nsub) load_rows(a, sm, b, h, grp, n0, len, k + 1, buf ^ 1, true);
        // the state entering sub-chunk k: lanes 0-63 forward rows, 64-127 flipped rows -> bf16 operands
        {
            const uint32_t lane_base = (uint32_t)(warp * 32);
            float t0[32], t1[32];
            tc::tmem_ld32(tc::tmem_addr(tmem, lane_base, k * 64), t0);
            tc::tmem_ld32(tc::tmem_addr(tmem, lane_base, k * 64 + 32), t1);
            tc::tmem_wait_ld();
            uint8_t *ht = warp < 2 ? sm.Hf() : sm.Hb();
            const int p = warp < 2 ? tid : tid - 64;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = t0[ch * 8 + e];
                put_chunk(ht, p, ch, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = t1[ch * 8 + e];
                put_chunk(ht, p, ch + 4, v);
            }
        }
        // factors of the decay matrix for this sub-chunk, around r = cum at its midpoint
        const int i = tid, n = k * kSub + i;
        const float ci = sm.cum()[n], di = sm.dt()[n];
        const float ei = ci - di * Ah;
        const float cend = sm.cum()[k * kSub + kSub - 1];
        const float r = sm.cum()[k * kSub + kSub / 2 - 1];
        sm.gf()[i] = __expf(r - ci) * di;   // forward column factor
        sm.gb()[i] = __expf(ei - r) * di;   // flipped column factor
        const float range = block_max128(fmaxf(fabsf(ci - r), fabsf(ei - r)), sm.red());
        const bool factored = range <= kFactorLimit;
        wait_loads(k + 1 < nsub);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // S = C B^T
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t idesc = tc::idesc_bf16(128, 128, 0, 0);
            const uint32_t c0 = tc::smem_u32(sm.C(buf)), b0 = tc::smem_u32(sm.B(buf));
#pragma unroll
            for (int s = 0; s < 4; ++s)
                tc::mma_bf16(tmem + kColS, tc::sdesc_sw128(c0 + s * 32, 16, 1024),
                             tc::sdesc_sw128(b0 + s * 32, 16, 1024), idesc, s > 0);
            tc::mma_commit(bar);
        }
        if (!mma_wait()) goto cleanup;

        // row i of A = [M | R_f C | R_b C]
        {
            const uint32_t lane_base = (uint32_t)(warp * 32);
            const float ff = __expf(ci - r);    // forward row factor
            const float fb = __expf(r - ei);    // flipped row factor
            for (int cc = 0; cc < 4; ++cc) {
                float sv[32];
                tc::tmem_ld32(tc::tmem_addr(tmem + kColS, lane_base, cc * 32), sv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = cc * 32 + q * 8 + e;
                        float w;
                        if (factored) {
                            w = (j <= i ? ff * sm.gf()[j] : 0.f) + (j >= i ? fb * sm.gb()[j] : 0.f);
                        } else {
                            const float cj = sm.cum()[k * kSub + j], dj = sm.dt()[k * kSub + j];
                            const float ej = cj - dj * Ah;
                            w = ((j <= i ? __expf(ci - cj) : 0.f) + (j >= i ? __expf(ej - ei) : 0.f)) * dj;
                        }
                        m[e] = sv[q * 8 + e] * w;
                    }
                    const int j0 = cc * 32 + q * 8;
                    put_chunk(sm.A(j0 >> 6), i, (j0 & 63) >> 3, m);
                }
            }
            const float rf = __expf(ci), rb = __expf(cend - ei);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float v[8], vf[8], vb[8];
                row_chunk(sm.C(buf), i, ch, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    vf[e] = rf * v[e];
                    vb[e] = rb * v[e];
                }
                put_chunk(sm.A(2), i, ch, vf);
                put_chunk(sm.A(3), i, ch, vb);
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // Acc = M x + (R_f C) h_f^T + (R_b C) h_b^T
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t id_mx = tc::idesc_bf16(128, 64, 0, 1);
            const uint32_t id_ch = tc::idesc_bf16(128, 64, 0, 0);
            const uint32_t a0 = tc::smem_u32(sm.A(0)), x0 = tc::smem_u32(sm.X(buf));
            const uint32_t hf = tc::smem_u32(sm.Hf()), hb = tc::smem_u32(sm.Hb());
#pragma unroll
            for (int s = 0; s < 8; ++s)
                tc::mma_bf16(tmem + kColAcc, tc::sdesc_sw128(a0 + (s >> 2) * kTile + (s & 3) * 32, 16, 1024),
                             tc::sdesc_sw128(x0 + s * 2048, kTile, 1024), id_mx, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                tc::mma_bf16(tmem + kColAcc, tc::sdesc_sw128(a0 + 2 * kTile + s * 32, 16, 1024),
                             tc::sdesc_sw128(hf + s * 32, 16, 1024), id_ch, true);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                tc::mma_bf16(tmem + kColAcc, tc::sdesc_sw128(a0 + 3 * kTile + s * 32, 16, 1024),
                             tc::sdesc_sw128(hb + s * 32, 16, 1024), id_ch, true);
            tc::mma_commit(bar);
        }
        if (!mma_wait()) goto cleanup;

        // epilogue: y_i = Acc_i + 2 D x_i -> grid position of token i. The TMEM loads are
        // warp-collective, so every lane issues them; only lanes of real tokens store.
        {
            const uint32_t lane_base = (uint32_t)(warp * 32);
            const bool valid = n < len;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out) +
                                 (((size_t)b * a.N + (valid ? sm.goff()[n] : 0)) * a.nh + h) * 64;
            for (int half = 0; half < 2; ++half) {
                float acc[32];
                tc::tmem_ld32(tc::tmem_addr(tmem + kColAcc, lane_base, half * 32), acc);
                tc::tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float xv[8], y[8];
                        row_chunk(sm.X(buf), i, half * 4 + q, xv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = acc[q * 8 + e] + 2.f * Dh * xv[e];
                        uint4 u;
                        u.x = tc::pack_bf16(y[0], y[1]);
                        u.y = tc::pack_bf16(y[2], y[3]);
                        u.z = tc::pack_bf16(y[4], y[5]);
                        u.w = tc::pack_bf16(y[6], y[7]);
                        *reinterpret_cast<uint4 *>(dst + half * 32 + q * 8) = u;
                    }
                }
            }
        }
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
    }

cleanup:
    tc::cp_async_wait_all();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool ssd_tc_supported(const SsdArgs &a)
{
    return a.bf16 && a.P == 64 && a.Ns == 64 && a.dirs == MATE_DIR_BI && a.Q % kSub == 0 && a.Q / kSub >= 1 &&
           a.Q / kSub <= kMaxSubs && a.nchunks <= 65535 && a.nh <= 65535 && a.batch <= 65535;
}

cudaError_t launch_ssd_tc(const SsdArgs &a, cudaStream_t s)
{
    cudaError_t e = cudaFuncSetAttribute(ssd_chunk_out_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_ssd_prepass_bf16_64(a, s);
    if (e != cudaSuccess) return e;
    Phase ph(MATE_PHASE_CHUNK_OUT, s);
    ssd_chunk_out_tc_kernel<<<dim3(a.nh, a.nchunks, a.batch), kThreads, kSmemBytes, s>>>(a, a.Q / kSub);
    return cudaGetLastError();
}

}  // namespace mate
