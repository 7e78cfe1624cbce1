// Bidirectional SSD scan on the 5th-generation tensor cores (tcgen05 + TMEM)
// for bf16 storage, head dim 64, d_state 64.
//
// Method (paper review "LinGen ...", section 三, MA-Branch items 1-2): per
// head, the Mamba2 recurrence s_n = exp(dt_n A) s_{n-1} + dt_n x_n B_n^T,
// y_n = s_n C_n + D x_n, over the Rotary-Major-Scan sequence and over its
// flip, flipped back and added. The RMS order enters only through gather
// addresses: row j of a chunk is the grid token of scan position start + j.
//
// Three kernels, all with one CTA per (head, chunk of L = 128*K tokens, batch
// element) where a chunk is processed as K sub-chunks of 128 tokens:
//
// chunk_state  chunk-local states of both directions from a zero start,
//              one accumulating MMA per sub-chunk
//                  [ (w_f x)^T ; (w_b x)^T ] (128 x 128 tokens) . B (128 tokens x 64)
//              with w_f[j] = exp(c_end - c_j) dt_j and w_b[j] = exp(e_j) dt_j
//              (c, e: inclusive / exclusive cumulative sums of A dt over the
//              chunk); rows 0-63 forward, rows 64-127 flipped.
// state_chain  one thread per 8 state elements replaces every chunk-local state
//              by the state entering the chunk (forward from the left, flipped
//              from the right), starting from the review state or zero. The
//              chunk states are stored as bf16 (halving their traffic); the
//              chain accumulates in fp32.
// chunk_out    phase 1: the same MMA per sub-chunk with sub-chunk-local
//              weights, each result kept in its own TMEM slot;
//              phase 2: chain the slots in TMEM from the chunk's entering
//              states (each lane owns a state row; forward lanes walk left to
//              right, flipped lanes right to left);
//              phase 3: per sub-chunk, S = C B^T (128 x 128) into TMEM; row i
//              of S becomes row i of A = [ M | R_f C | R_b C ] (128 x 256) with
//                  M_ij = S_ij dt_j (exp(c_i - c_j) [j <= i] + exp(e_j - e_i) [j >= i]),
//                  R_f[i] = exp(c_i), R_b[i] = exp(c_end - e_i),
//              and one accumulating MMA chain computes A . [ x ; h_f^T ; h_b^T ]
//              (M as bf16 pairs in TMEM over S, read there as the A operand);
//              the epilogue adds 2 D x and stores each row at its grid position.
// The exponentials of M are factored around the sub-chunk midpoint r,
// exp(c_i - c_j) = exp(c_i - r) exp(r - c_j), whenever the sub-chunk's decay
// range fits fp32; otherwise every element is exponentiated exactly.
//
// 256 threads per CTA: thread t works on row r = t % 128 (TMEM lane r) and
// half g = t / 128 of that row's columns.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace mate {

namespace {

constexpr int kThreads = 256;
constexpr int kSub = 128;        // tokens per sub-chunk
constexpr int kMaxSubs = 4;      // sub-chunks per chunk held in TMEM
constexpr int kMaxChunk = kSub * kMaxSubs;
constexpr uint32_t kTile = 16384;

constexpr float kFactorLimit = 80.f;  // |exponent| bound for the factored exps

// ---------------------------------------------------------------------------
// helpers shared by the kernels
// ---------------------------------------------------------------------------

// Gather the 128 token rows of sub-chunk `sub` into swizzled tiles (x: the 64
// head dims of head h; B and C: the 64 state dims of the head's group; tC may
// be null). goff[n] is the grid offset of chunk position n; rows past the
// sequence end are zero. Eight consecutive threads copy the eight 16-byte
// chunks of one row, so a warp reads four whole 128-byte rows.
__device__ __forceinline__ void load_rows(const SsdArgs &a, uint8_t *tX, uint8_t *tB, uint8_t *tC, const int *goff,
                                          int b, int h, int grp, int len, int sub)
{
    const int c = threadIdx.x & 7;
    const char *xb = static_cast<const char *>(a.x) + ((size_t)h * 64 + c * 8) * 2;
    const size_t gb = ((size_t)grp * 64 + c * 8) * 2;
    const char *bb = static_cast<const char *>(a.B) + gb;
    const char *cb = static_cast<const char *>(a.C) + gb;
#pragma unroll
    for (int q = 0; q < kSub / (kThreads / 8); ++q) {
        const int r = (threadIdx.x >> 3) + q * (kThreads / 8);
        const int n = sub * kSub + r;
        const uint32_t off = tc::sw128(r, c);
        if (n < len) {
            const size_t tok = (size_t)b * a.N + goff[n];
            tc::cp_async16(tX + off, xb + tok * (size_t)a.nh * 128);
            tc::cp_async16(tB + off, bb + tok * (size_t)a.G * 128);
            if (tC) tc::cp_async16(tC + off, cb + tok * (size_t)a.G * 128);
        } else {
            const uint4 z = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(tX + off) = z;
            *reinterpret_cast<uint4 *>(tB + off) = z;
            if (tC) *reinterpret_cast<uint4 *>(tC + off) = z;
        }
    }
    tc::cp_async_commit();
}

// Where the scan order makes every 128-position sub-chunk a box of the grid,
// its x, B, C rows come by TMA (one box each, already in the 128-byte swizzle)
// instead of per-thread gathers. One kernel launch per batch element then.
struct TmaRows {
    int use;      // 1: TMA boxes
    int n0, n1;   // scan axis lengths, fastest first
    int zbase;    // batch element of blockIdx.z == 0
};

// issued by one thread: x (channel h) and B, C (channel grp; tC may be null) rows
// of the sub-chunk starting at scan position s, completing on `bar`
__device__ __forceinline__ void tma_rows(const CUtensorMap *mx, const CUtensorMap *mb, const CUtensorMap *mc,
                                         const TmaRows &g, uint8_t *tX, uint8_t *tB, uint8_t *tC, uint64_t *bar,
                                         int h, int grp, int s)
{
    const int a0 = s % g.n0, q = s / g.n0, a1 = q % g.n1, a2 = q / g.n1;
    tc::mbar_expect_tx(bar, (tC ? 3u : 2u) * kTile);
    tc::tma_load_5d(tX, mx, bar, 0, h, a0, a1, a2);
    tc::tma_load_5d(tB, mb, bar, 0, grp, a0, a1, a2);
    if (tC) tc::tma_load_5d(tC, mc, bar, 0, grp, a0, a1, a2);
}

__device__ __forceinline__ void wait_loads(bool newer_pending)
{
    if (newer_pending)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
    else
        asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// rms_grid_offset with the divisions by T, H, W and H*W taken by the launch-time
// FastDiv divisors (scan positions and grid offsets are below 2^31).
__device__ __forceinline__ int rms_offset_fast(int n, const SsdArgs &a)
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
    case MATE_SCAN_ZZ: {  // 3D boustrophedon (mate.h)
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

// Per-chunk setup shared by chunk_state and chunk_out: grid offsets and dt of
// the chunk's L positions (zero past the sequence end).
__device__ __forceinline__ void load_chunk_meta(const SsdArgs &a, int b, int h, int n0, int len, int L, int *goff,
                                                float *dt)
{
    for (int n = threadIdx.x; n < L; n += kThreads) {
        float d = 0.f;
        int g = 0;
        if (n < len) {
            g = rms_offset_fast(n0 + n, a);
            d = a.dt[((size_t)b * a.N + g) * a.nh + h];
        }
        goff[n] = g;
        dt[n] = d;
    }
}

// Grid offsets of the chunk's L positions (0 past the sequence end).
__device__ __forceinline__ void chunk_offsets(const SsdArgs &a, int n0, int len, int L, int *goff)
{
    for (int n = threadIdx.x; n < L; n += kThreads) goff[n] = n < len ? rms_offset_fast(n0 + n, a) : 0;
}

// Inclusive cumulative sums of A*dt within each 128-token sub-chunk (warp w
// scans sub-chunk w); with `chunk_level`, continued across sub-chunks.
__device__ __forceinline__ void sub_cumsums(const float *dt, float *cum, float Ah, int nsub, bool chunk_level,
                                            float *carry_out)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < nsub) {
        float carry = 0.f;
        for (int q = 0; q < kSub; q += 32) {
            const int n = warp * kSub + q + lane;
            const float v = warp_inclusive_scan(dt[n] * Ah) + carry;
            cum[n] = v;
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) carry_out[warp] = carry;
    }
    __syncthreads();
    if (chunk_level) {
        for (int n = threadIdx.x; n < nsub * kSub; n += kThreads) {
            float off = 0.f;
            for (int w = 0; w < n / kSub; ++w) off += carry_out[w];
            cum[n] += off;
        }
        __syncthreads();
    }
}

// U_f row r = w_f[r] x_r and U_b row r = w_b[r] x_r for chunks [4g, 4g + 4), as
// packed bf16 products (w rounded to bf16 once; each product rounded once).
__device__ __forceinline__ __nv_bfloat162 bf16x2_of(uint32_t u) { return *reinterpret_cast<__nv_bfloat162 *>(&u); }
__device__ __forceinline__ uint32_t u32_of(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }

__device__ __forceinline__ uint4 scale_chunk(uint4 x, __nv_bfloat162 w)
{
    return make_uint4(u32_of(__hmul2(bf16x2_of(x.x), w)), u32_of(__hmul2(bf16x2_of(x.y), w)),
                      u32_of(__hmul2(bf16x2_of(x.z), w)), u32_of(__hmul2(bf16x2_of(x.w), w)));
}

__device__ __forceinline__ void build_u(const uint8_t *tX, uint8_t *uf, uint8_t *ub, int r, int g, float wf, float wb)
{
    const __nv_bfloat162 f2 = __float2bfloat162_rn(wf), b2 = __float2bfloat162_rn(wb);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t off = tc::sw128(r, 4 * g + q);
        const uint4 x = *reinterpret_cast<const uint4 *>(tX + off);
        *reinterpret_cast<uint4 *>(uf + off) = scale_chunk(x, f2);
        *reinterpret_cast<uint4 *>(ub + off) = scale_chunk(x, b2);
    }
}

// [U_f^T ; U_b^T] (MN-major, two 64-row groups) . B (MN-major), K = 128 tokens
__device__ __forceinline__ void mma_states(uint32_t d_tmem, uint32_t uf_addr, uint32_t b_addr, bool accumulate)
{
    const uint32_t idesc = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
    for (int s = 0; s < 8; ++s)
        tc::mma_bf16(d_tmem, tc::sdesc_sw128(uf_addr + s * 2048, kTile, 1024),
                     tc::sdesc_sw128(b_addr + s * 2048, kTile, 1024), idesc, accumulate || s > 0);
}

// Bounded wait for the next MMA completion on `bar`: warp 0 polls the barrier
// while the other warps wait at __syncthreads (no issue slots spent). On
// timeout every thread returns false, after a second bounded wait for the MMAs
// in flight.
__device__ __forceinline__ bool mma_wait(uint64_t *bar, uint32_t &phase, int *err, int *abort_flag)
{
    if ((threadIdx.x >> 5) == 0) {
        const bool ok = tc::mbar_wait(bar, phase & 1u, err);
        if (!ok && threadIdx.x == 0) *abort_flag = 1;
    }
    ++phase;
    __syncthreads();
    if (*abort_flag) {
        if (threadIdx.x == 0) tc::mbar_wait(bar, (phase - 1) & 1u, nullptr);
        __syncthreads();
        return false;
    }
    tc::tc_fence_after();
    return true;
}

// ---------------------------------------------------------------------------
// chunk_out: ~101 KB of shared memory, 256 TMEM columns and at most 128
// registers per thread, so two CTAs share an SM.
//   TMEM columns   0..127 : the K sub-chunk states, packed bf16 (32 columns each:
//                           64 values of a state row per lane)
//   TMEM columns 128..255 : phase 1 MMA result (64 cols), phase 3 S (128 cols),
//                           then M as bf16 pairs (columns 0-31 and 96-127 of the
//                           region) and the output accumulator (columns 32-95)
//   shared memory         : x, B, C tiles of one sub-chunk; two 16 KB tiles for
//                           U_f / U_b (phase 1) or the epilogue's staging (phase 3);
//                           h_f, h_b operands.
//                           In phase 3, R_f C overwrites the C tile and R_b C the
//                           B tile once S = C B^T is done.
// Loads overlap math: phase 1 double-buffers x, B in the {x, B} and {C, h}
// tiles; the chunk's entering states arrive during the last phase-1 sub-chunk;
// the first output sub-chunk's rows load during phase 2 and each later one's
// during the previous epilogue (x kept in registers for the 2 D x term).
// ---------------------------------------------------------------------------
constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffB = kTile;
constexpr uint32_t kOffC = 2 * kTile;
constexpr uint32_t kOffM = 3 * kTile;       // 2 tiles: U_f, U_b / M0, M1
constexpr uint32_t kOffH = 5 * kTile;       // h_f (8 KB) then h_b (8 KB)
constexpr uint32_t kOffDt = 6 * kTile;                // 2 x dt[512]: this item's, the next item's
constexpr uint32_t kOffCum = kOffDt + 2 * kMaxChunk * 4;
constexpr uint32_t kOffGoff = kOffCum + kMaxChunk * 4;
constexpr uint32_t kOffGf = kOffGoff + kMaxChunk * 4;
constexpr uint32_t kOffGb = kOffGf + kMaxChunk * 4;
constexpr uint32_t kOffRed = kOffGb + kMaxChunk * 4;  // 8 floats
constexpr uint32_t kOffFlag = kOffRed + 32;           // kMaxSubs ints: sub-chunk takes the factored exps
constexpr uint32_t kOffBar = kOffRed + 64;
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;  // bar, TMEM slot, abort flag, ldbar, dtbar
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "chunk_out: two CTAs per SM");

constexpr uint32_t kColR = 128;   // scratch region after the packed state slots
constexpr uint32_t kTmemCols = 256;

__device__ __forceinline__ uint32_t bf2(float lo, float hi) { return tc::pack_bf16(lo, hi); }

__global__ void __launch_bounds__(kThreads, 2)
    ssd_chunk_out_tc_kernel(SsdArgs a, int nsub, const __grid_constant__ CUtensorMap mx,
                            const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mC,
                            const __grid_constant__ CUtensorMap mO, TmaRows geo, int nitems)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t *sX = base + kOffX, *sB = base + kOffB, *sC = base + kOffC, *sM = base + kOffM;
    uint8_t *sHf = base + kOffH, *sHb = base + kOffH + 8192;
    float *sdt_buf = reinterpret_cast<float *>(base + kOffDt);
    float *scum = reinterpret_cast<float *>(base + kOffCum);
    int *sgoff = reinterpret_cast<int *>(base + kOffGoff);
    float *sgf = reinterpret_cast<float *>(base + kOffGf);
    float *sgb = reinterpret_cast<float *>(base + kOffGb);
    float *sred = reinterpret_cast<float *>(base + kOffRed);
    int *sflag = reinterpret_cast<int *>(base + kOffFlag);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffBar + 8);
    int *abort_flag = reinterpret_cast<int *>(base + kOffBar + 12);
    uint64_t *ldbar = reinterpret_cast<uint64_t *>(base + kOffBar + 16);  // TMA row loads
    uint64_t *dtbar = reinterpret_cast<uint64_t *>(base + kOffBar + 24);  // dt of an item

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & (kSub - 1), g = tid >> 7;   // row / TMEM lane, column half
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
    const int L = nsub * kSub;
    uint32_t ld_issued = 0, ld_phase = 0;  // TMA batches issued / completed
    uint32_t dt_issued = 0, dt_phase = 0;  // dt loads issued / completed
    uint32_t mma_phase = 0;                // MMA completions on bar
    // the work item in hand: head h of chunk c of batch element b (heads fastest)
    int h = 0, c = 0, b = 0, n0 = 0, len = 0, grp = 0;
    float Ah = 0.f, Dh2 = 0.f;
    // dt of item `it` (written in scan order by chunk_state) into dt buffer `buf`,
    // completing on dtbar; issued by one thread
    auto issue_dt = [&](int it, int buf) {
        const int ih = it % a.nh, ic = (it / a.nh) % a.nchunks, ib = it / (a.nh * a.nchunks) + geo.zbase;
        tc::mbar_expect_tx(dtbar, (uint32_t)L * 4u);
        tc::bulk_load(sdt_buf + buf * kMaxChunk, a.dt_scan + (((size_t)ib * a.nh + ih) * a.nchunks + ic) * L,
                      (uint32_t)L * 4u, dtbar);
    };

    if (warp == 0) tc::tmem_alloc(tmem_slot, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(ldbar, 1);
        tc::mbar_init(dtbar, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
        if ((int)blockIdx.x < nitems) issue_dt(blockIdx.x, 0);
    }
    if ((int)blockIdx.x < nitems) ++dt_issued;
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tR = tmem + kColR;
    // rows of sub-chunk `sub` into the given tiles: a TMA batch from one thread, or
    // per-thread cp.async gathers
    auto issue_rows = [&](uint8_t *tx, uint8_t *tb, uint8_t *tcc, int sub) {
        if (geo.use) {
            if (tid == 0) tma_rows(&mx, &mB, &mC, geo, tx, tb, tcc, ldbar, h, grp, n0 + sub * kSub);
            ++ld_issued;
        } else {
            load_rows(a, tx, tb, tcc, sgoff, b, h, grp, len, sub);
        }
    };
    // waits for the pending TMA batch (at most one) and every cp.async group, then a
    // CTA barrier; false (on every thread) once a wait has timed out
    auto rows_wait = [&]() {
        if (ld_issued > ld_phase) {
            if (tc::mbar_wait(ldbar, ld_phase & 1u, a.err))
                ++ld_phase;
            else
                *abort_flag = 1;
        }
        tc::cp_async_wait_all();
        __syncthreads();
        return *abort_flag == 0;
    };
    // persistent: this CTA takes items blockIdx.x, + gridDim.x, ...
    for (int item = blockIdx.x, li = 0; item < nitems; item += gridDim.x, ++li) {
    h = item % a.nh;
    c = (item / a.nh) % a.nchunks;
    b = item / (a.nh * a.nchunks) + geo.zbase;
    n0 = c * L;
    len = min(L, a.N - n0);
    grp = h / (a.nh / a.G);
    Ah = a.A[h];
    Dh2 = 2.f * a.D[h];
    float *sdt = sdt_buf + (li & 1) * kMaxChunk;
    if (tid == 0 && geo.use) {
        // TMA boxes need no grid offsets: sub-chunk 0's rows are requested first
        tma_rows(&mx, &mB, &mC, geo, sX, sB, nullptr, ldbar, h, grp, n0);
        // the output phase reads x and B again (from L2, read in phase 1) and C for
        // the first time: C of every sub-chunk into L2 now
        for (int k = 0; k < nsub; ++k) {
            const int sp = n0 + k * kSub, a0 = sp % geo.n0, q = sp / geo.n0;
            tc::tma_prefetch_5d(&mC, 0, grp, a0, q % geo.n1, q / geo.n1);
        }
    }
    if (geo.use) ++ld_issued;
    else chunk_offsets(a, n0, len, L, sgoff);  // the gathers need the grid offsets
    // this item's dt (requested during the previous item, or at the start)
    if (!tc::mbar_wait(dtbar, dt_phase & 1u, a.err)) *abort_flag = 1;
    ++dt_phase;
    __syncthreads();
    if (*abort_flag) goto cleanup;
    // x, B of sub-chunk 0 are in flight while the decay factors are prepared
    if (!geo.use) issue_rows(sX, sB, nullptr, 0);  // (the TMA batch is already in flight)
    sub_cumsums(sdt, scum, Ah, nsub, false, sred);
    // warp k: column factors of sub-chunk k around its midpoint r_k,
    //   gf[n] = exp(r_k - c_n) dt_n, gb[n] = exp(e_n - r_k) dt_n,
    // and whether every factor exponent of the sub-chunk stays within the limit
    if (warp < nsub) {
        const float rmid = scum[warp * kSub + kSub / 2 - 1];
        float range = 0.f;
#pragma unroll
        for (int q = 0; q < kSub / 32; ++q) {
            const int n = warp * kSub + q * 32 + lane;
            const float cn = scum[n], dn = sdt[n], en = cn - dn * Ah;
            sgf[n] = __expf(rmid - cn) * dn;
            sgb[n] = __expf(en - rmid) * dn;
            range = fmaxf(range, fmaxf(fabsf(cn - rmid), fabsf(en - rmid)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) range = fmaxf(range, __shfl_xor_sync(0xffffffffu, range, o));
        if (lane == 0) sflag[warp] = range <= kFactorLimit;
    }

    // ---------------- phase 1: sub-chunk-local states -> packed bf16 slots ------------
    // x and B of sub-chunk k sit in buffer k % 2 ({x, B} tiles or {C, h} tiles);
    // the next sub-chunk's rows load while this one is processed.
    if (!rows_wait()) goto cleanup;
    for (int k = 0; k < nsub; ++k) {
        uint8_t *tx = (k & 1) ? sC : sX, *tb = (k & 1) ? sHf : sB;
        if (k + 1 < nsub) {
            // buffer (k + 1) % 2 was last read by sub-chunk k - 1, whose MMA is done
            issue_rows((k & 1) ? sX : sC, (k & 1) ? sB : sHf, nullptr, k + 1);
        } else {
            // the chunk's entering states (fwd rows 0-63, flipped rows 64-127) into
            // the free buffer's first tile: thread (r, g) copies its 64 bytes
            const bool fwd = r < 64;
            const char *Hin = reinterpret_cast<const char *>(fwd ? a.states_f : a.states_b) +
                              (((((size_t)b * a.nh + h) * a.nchunks + c) * 64 + (r & 63)) * 64 + 32 * g) * 2;
            uint8_t *dst = ((k & 1) ? sX : sC) + r * 128 + g * 64;
#pragma unroll
            for (int q = 0; q < 4; ++q) tc::cp_async16(dst + 16 * q, Hin + 16 * q);
            tc::cp_async_commit();
        }
        {
            const int n = k * kSub + r;
            const float cj = scum[n], dj = sdt[n], cend = scum[k * kSub + kSub - 1];
            build_u(tx, sM, sM + kTile, r, g, __expf(cend - cj) * dj, __expf(cj - dj * Ah) * dj);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            mma_states(tR, tc::smem_u32(sM), tc::smem_u32(tb), false);
            tc::mma_commit(bar);
        }
        if (!mma_wait(bar, mma_phase, a.err, abort_flag)) goto cleanup;
        {
            // fp32 result columns 32g .. 32g+31 of row r -> 16 packed columns of slot k
            float v[32];
            tc::tmem_ld32(tc::tmem_addr(tR, lane_base, 32 * g), v);
            tc::tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) pk[q] = bf2(v[2 * q], v[2 * q + 1]);
            tc::tmem_st16(tc::tmem_addr(tmem, lane_base, k * 32 + 16 * g), pk);
            tc::tmem_wait_st();
        }
        // the next sub-chunk's rows (or, after the last, the entering states) have landed
        tc::tc_fence_before();
        if (!rows_wait()) goto cleanup;
        tc::tc_fence_after();
    }

    // ---------------- phase 2: chain the sub-chunk states ------------------------------
    {
        const bool fwd = r < 64;
        float hv[32];
        {
            const uint8_t *src = ((nsub & 1) ? sC : sX) + r * 128 + g * 64;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 u = *reinterpret_cast<const uint4 *>(src + 16 * q);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = tc::unpack_bf16(w4[e]);
                    hv[8 * q + 2 * e] = f.x;
                    hv[8 * q + 2 * e + 1] = f.y;
                }
            }
        }
        tc::fence_proxy_async_smem();
        __syncthreads();
        // x, B, C of the first output sub-chunk load during the chain
        issue_rows(sX, sB, sC, 0);
        // two slots per TMEM round trip (loads of both, then stores of both)
        for (int it0 = 0; it0 < nsub; it0 += 2) {
            const bool two = it0 + 1 < nsub;
            const int k0 = fwd ? it0 : nsub - 1 - it0, k1 = fwd ? it0 + 1 : nsub - 2 - it0;
            uint32_t loc[2][16], pk[2][16];  // separate sources for the two stores in flight
            tc::tmem_ld16(tc::tmem_addr(tmem, lane_base, k0 * 32 + 16 * g), loc[0]);
            if (two) tc::tmem_ld16(tc::tmem_addr(tmem, lane_base, k1 * 32 + 16 * g), loc[1]);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (u == 1 && !two) break;
                const int k = u == 0 ? k0 : k1;
                const float alpha = __expf(scum[k * kSub + kSub - 1]);
#pragma unroll
                for (int q = 0; q < 16; ++q) pk[u][q] = bf2(hv[2 * q], hv[2 * q + 1]);
                tc::tmem_st16(tc::tmem_addr(tmem, lane_base, k * 32 + 16 * g), pk[u]);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float2 hn = tc::fma_f32x2(make_float2(alpha, alpha), make_float2(hv[2 * q], hv[2 * q + 1]),
                                                    tc::unpack_bf16(loc[u][q]));
                    hv[2 * q] = hn.x, hv[2 * q + 1] = hn.y;
                }
            }
            tc::tmem_wait_st();
        }
    }

    // ---------------- phase 3: outputs ---------------------------------------------
    // Four barriers per sub-chunk: S done, M and R C written, Acc done (x rows read,
    // so the next rows may load), and the epilogue done with the next rows landed.
    //
    // entering states of sub-chunk kk (already bf16) -> operand rows (forward if r < 64);
    // each thread moves its own TMEM lane and columns
    {
    auto write_h = [&](int kk) {
        uint32_t pk[16];
        tc::tmem_ld16(tc::tmem_addr(tmem, lane_base, kk * 32 + 16 * g), pk);
        tc::tmem_wait_ld();
        uint8_t *ht = r < 64 ? sHf : sHb;
        const int p = r & 63;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(ht + tc::sw128(p, 4 * g + q)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    };
    write_h(0);
    if (item + (int)gridDim.x < nitems) {
        // the next item's dt into the other buffer (last read by the item before this
        // one), and its first rows into L2
        if (tid == 0) {
            const int nx = item + gridDim.x;
            issue_dt(nx, (li + 1) & 1);
            if (geo.use) {
                const int nh_ = nx % a.nh, nc = (nx / a.nh) % a.nchunks, sp = nc * L;
                const int a0 = sp % geo.n0, q = sp / geo.n0;
                tc::tma_prefetch_5d(&mx, 0, nh_, a0, q % geo.n1, q / geo.n1);
                tc::tma_prefetch_5d(&mB, 0, nh_ / (a.nh / a.G), a0, q % geo.n1, q / geo.n1);
            }
        }
        ++dt_issued;
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    if (!rows_wait()) goto cleanup;
    for (int k = 0; k < nsub; ++k) {
        const int n = k * kSub + r;
        const float ci = scum[n], di = sdt[n];
        const float ei = ci - di * Ah;
        const float cend = scum[k * kSub + kSub - 1];
        const float rmid = scum[k * kSub + kSub / 2 - 1];
        const float *gf = sgf + k * kSub, *gb = sgb + k * kSub;  // column factors of this sub-chunk
        const bool factored = sflag[k] != 0;

        // S = C B^T -> TMEM R
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t idesc = tc::idesc_bf16(128, 128, 0, 0);
            const uint32_t c0 = tc::smem_u32(sC), b0 = tc::smem_u32(sB);
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2)
                tc::mma_bf16(tR, tc::sdesc_sw128(c0 + s2 * 32, 16, 1024), tc::sdesc_sw128(b0 + s2 * 32, 16, 1024), idesc,
                             s2 > 0);
            tc::mma_commit(bar);
        }
        if (!mma_wait(bar, mma_phase, a.err, abort_flag)) goto cleanup;

        // row r of M: the thread's S columns, 16 of each 32-column block b (columns
        // 32b + 16g ..), times the decay factors; each warp's diagonal block is thus
        // split evenly between the row's two threads. The bf16 pairs of block b go to
        // TMEM columns 32(b/2) + 16g + 8(b%2) of R (columns 0-63, S columns this thread
        // has already read), where the output MMA reads M as its A operand.
        {
            const float ff = __expf(ci - rmid), fb = __expf(rmid - ei);
            const int wq = warp & 3;  // this warp's rows are 32*wq .. 32*wq + 31
#pragma unroll
            for (int qp = 0; qp < 4; qp += 2) {
                uint32_t raw2[2][16], mp[2][8];  // two 16-column TMEM loads per wait
                tc::tmem_ld16(tc::tmem_addr(tR, lane_base, 32 * qp + 16 * g), raw2[0]);
                tc::tmem_ld16(tc::tmem_addr(tR, lane_base, 32 * qp + 32 + 16 * g), raw2[1]);
                tc::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int j0 = 32 * (qp + u) + 16 * g;   // first of these 16 columns
                    float sv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) sv[e] = __uint_as_float(raw2[u][e]);
                    const int cc = j0 >> 5;                  // 32-column block of these columns
                    if (factored && cc != wq) {              // off the diagonal block: one direction only
                        // left of every row of this warp: forward; right of every row: flipped
                        const float4 *fac = reinterpret_cast<const float4 *>((cc < wq ? gf : gb) + j0);
                        const float rf = cc < wq ? ff : fb;
                        const float2 rf2 = make_float2(rf, rf);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {  // packed fp32 pairs
                            const float4 f4 = fac[q];
                            const float2 a = tc::mul_f32x2(make_float2(sv[4 * q], sv[4 * q + 1]),
                                                           tc::mul_f32x2(rf2, make_float2(f4.x, f4.y)));
                            const float2 c2 = tc::mul_f32x2(make_float2(sv[4 * q + 2], sv[4 * q + 3]),
                                                            tc::mul_f32x2(rf2, make_float2(f4.z, f4.w)));
                            sv[4 * q] = a.x, sv[4 * q + 1] = a.y, sv[4 * q + 2] = c2.x, sv[4 * q + 3] = c2.y;
                        }
                    } else if (factored) {                   // the diagonal block
                        const float4 *f4p = reinterpret_cast<const float4 *>(gf + j0);
                        const float4 *b4p = reinterpret_cast<const float4 *>(gb + j0);
                        const float2 ff2 = make_float2(ff, ff), fb2 = make_float2(fb, fb);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {  // packed fp32 pairs
                            const float4 f4 = f4p[q], b4 = b4p[q];
                            const float2 tf[2] = {tc::mul_f32x2(ff2, make_float2(f4.x, f4.y)),
                                                  tc::mul_f32x2(ff2, make_float2(f4.z, f4.w))};
                            const float2 tb[2] = {tc::mul_f32x2(fb2, make_float2(b4.x, b4.y)),
                                                  tc::mul_f32x2(fb2, make_float2(b4.z, b4.w))};
#pragma unroll
                            for (int e2 = 0; e2 < 2; ++e2) {
                                const int j = j0 + 4 * q + 2 * e2;
                                const float2 w = make_float2((j <= r ? tf[e2].x : 0.f) + (j >= r ? tb[e2].x : 0.f),
                                                             (j + 1 <= r ? tf[e2].y : 0.f) + (j + 1 >= r ? tb[e2].y : 0.f));
                                const float2 m = tc::mul_f32x2(make_float2(sv[4 * q + 2 * e2], sv[4 * q + 2 * e2 + 1]), w);
                                sv[4 * q + 2 * e2] = m.x, sv[4 * q + 2 * e2 + 1] = m.y;
                            }
                        }
                    } else {                                 // decay range too wide: exact exponentials
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int j = j0 + e;
                            const float cj = scum[k * kSub + j], dj = sdt[k * kSub + j];
                            const float ej = cj - dj * Ah;
                            sv[e] *= ((j <= r ? __expf(ci - cj) : 0.f) + (j >= r ? __expf(ej - ei) : 0.f)) * dj;
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) mp[u][e] = bf2(sv[2 * e], sv[2 * e + 1]);
                }
                tc::tmem_st8(tc::tmem_addr(tR, lane_base, 16 * qp + 16 * g), mp[0]);
                tc::tmem_st8(tc::tmem_addr(tR, lane_base, 16 * qp + 16 * g + 8), mp[1]);
            }
            tc::tmem_wait_st();
        }
        {
            // C row r, chunks 4g .. 4g+3 (this thread's own): R_f C over the C tile and
            // R_b C over the B tile (free once S is done), in the same positions
            const __nv_bfloat162 rf = __float2bfloat162_rn(__expf(ci)), rb = __float2bfloat162_rn(__expf(cend - ei));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = tc::sw128(r, 4 * g + q);
                const uint4 cv = *reinterpret_cast<const uint4 *>(sC + off);
                *reinterpret_cast<uint4 *>(sC + off) = scale_chunk(cv, rf);
                *reinterpret_cast<uint4 *>(sB + off) = scale_chunk(cv, rb);
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // Acc = M x + (R_f C) h_f^T + (R_b C) h_b^T -> TMEM R columns 64..127 (S there is
        // consumed); M comes from TMEM: K-step s (tokens 16s ..) is block s/2 of thread
        // g = s%2, at column 32(s/4) + 16(s%2) + 8((s/2)%2)
        const uint32_t tAcc = tR + 64;
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t id_mx = tc::idesc_bf16(128, 64, 0, 1);
            const uint32_t id_ch = tc::idesc_bf16(128, 64, 0, 0);
            const uint32_t x0 = tc::smem_u32(sX);
            const uint32_t cf = tc::smem_u32(sC), cb = tc::smem_u32(sB);
            const uint32_t hf = tc::smem_u32(sHf), hb = tc::smem_u32(sHb);
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                tc::mma_bf16_tmem_a(tAcc, tR + 32 * (s2 >> 2) + 16 * (s2 & 1) + 8 * ((s2 >> 1) & 1),
                                    tc::sdesc_sw128(x0 + s2 * 2048, kTile, 1024), id_mx, s2 > 0);
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2)
                tc::mma_bf16(tAcc, tc::sdesc_sw128(cf + s2 * 32, 16, 1024), tc::sdesc_sw128(hf + s2 * 32, 16, 1024),
                             id_ch, true);
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2)
                tc::mma_bf16(tAcc, tc::sdesc_sw128(cb + s2 * 32, 16, 1024), tc::sdesc_sw128(hb + s2 * 32, 16, 1024),
                             id_ch, true);
            tc::mma_commit(bar);
        }
        // this row's x (for the 2 D x term) to registers while the MMA runs (reads only)
        uint4 xr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xr[q] = *reinterpret_cast<const uint4 *>(sX + tc::sw128(r, 4 * g + q));
        tc::fence_proxy_async_smem();  // those reads precede the next rows' TMA writes
        if (!mma_wait(bar, mma_phase, a.err, abort_flag)) goto cleanup;

        // every tile is free: the next sub-chunk's states go to the h tiles and its
        // x, B, C load while the epilogue runs
        if (k + 1 < nsub) {
            write_h(k + 1);
            issue_rows(sX, sB, sC, k + 1);
        }

        // epilogue: columns 32g .. 32g+31 of y_r = Acc_r + 2 D x_r, rounded to bf16
        {
            uint32_t acc2[2][16];
            tc::tmem_ld16(tc::tmem_addr(tAcc, lane_base, 32 * g), acc2[0]);
            tc::tmem_ld16(tc::tmem_addr(tAcc, lane_base, 32 * g + 16), acc2[1]);
            tc::tmem_wait_ld();
            // 16-byte chunk q of this thread's half row (eight bf16 values)
            auto chunk16 = [&](int q) {
                const uint32_t *acc = acc2[q >> 1] + 8 * (q & 1);
                const uint32_t xw[4] = {xr[q].x, xr[q].y, xr[q].z, xr[q].w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 y2 = tc::fma_f32x2(make_float2(Dh2, Dh2), tc::unpack_bf16(xw[e]),
                                                    make_float2(__uint_as_float(acc[2 * e]),
                                                                __uint_as_float(acc[2 * e + 1])));
                    o4[e] = bf2(y2.x, y2.y);
                }
                return make_uint4(o4[0], o4[1], o4[2], o4[3]);
            };
            if (geo.use) {
                // the sub-chunk's rows form one box of the grid: stage them in the 128-byte
                // swizzle (one of the two free M tiles, alternating) and store the box by TMA;
                // rows past the sequence end fall outside the tensor and are not written
                uint8_t *stg = sM + (k & 1) * kTile;
#pragma unroll
                for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4 *>(stg + tc::sw128(r, 4 * g + q)) = chunk16(q);
                tc::fence_proxy_async_smem();
                __syncthreads();
                if (tid == 0) {
                    const int sp = n0 + k * kSub, a0 = sp % geo.n0, qq = sp / geo.n0;
                    tc::tma_store_5d(&mO, stg, 0, h, a0, qq % geo.n1, qq / geo.n1);
                    tc::bulk_commit();
                    // the store before this one has read its tile, which the next
                    // sub-chunk's epilogue writes (after the barriers in between)
                    tc::bulk_wait_read<1>();
                }
            } else {
                // each warp stages its 32 half rows (64 bytes) in its own 2 KB of the free M
                // tiles, then stores them at the grid positions of their tokens, eight half
                // rows per store instruction
                uint8_t *stg = sM + warp * 2048;
                const int lr = r & 31;  // this thread's row within the warp
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(stg + lr * 64 + ((q ^ ((lr >> 1) & 3)) << 4)) = chunk16(q);
                __syncwarp();
                const int row0 = r & ~31;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = i * 8 + (lane >> 2), q = lane & 3, nn = k * kSub + row0 + rr;
                    if (nn < len) {
                        const uint4 v =
                            *reinterpret_cast<const uint4 *>(stg + rr * 64 + ((q ^ ((rr >> 1) & 3)) << 4));
                        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out) +
                                             (((size_t)b * a.N + sgoff[nn]) * a.nh + h) * 64 + 32 * g + q * 8;
                        *reinterpret_cast<uint4 *>(dst) = v;
                    }
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        if (!rows_wait()) goto cleanup;
        tc::tc_fence_after();
    }
    }
    // the next item's phase 1 writes the M tiles, which the last output stores read
    if (tid == 0) tc::bulk_wait_read<0>();
    // this item's dt buffer is written next by a bulk load (async proxy)
    tc::fence_proxy_async_smem();
    __syncthreads();
    }

cleanup:
    tc::cp_async_wait_all();
    // after a timeout a TMA batch or a dt load may still be landing: bounded waits for them
    if (ld_issued > ld_phase && tid == 0) tc::mbar_wait(ldbar, ld_phase & 1u, nullptr);
    if (dt_issued > dt_phase && tid == 0) tc::mbar_wait(dtbar, dt_phase & 1u, nullptr);
    if (tid == 0) tc::bulk_wait_all();  // output stores read shared memory until they complete
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// chunk_state: ~54 KB of shared memory and 64 TMEM columns, so four CTAs
// share an SM and their loads overlap each other's math. U_f is written over
// the x tile it is computed from.
// ---------------------------------------------------------------------------
constexpr uint32_t kStOffX = 0;            // x, then U_f
constexpr uint32_t kStOffU = kTile;        // U_b (right after U_f: the MMA's second M group)
constexpr uint32_t kStOffB = 2 * kTile;
constexpr uint32_t kStOffDt = 3 * kTile;
constexpr uint32_t kStOffCum = kStOffDt + kMaxChunk * 4;
constexpr uint32_t kStOffGoff = kStOffCum + kMaxChunk * 4;
constexpr uint32_t kStOffRed = kStOffGoff + kMaxChunk * 4;  // 8 floats
constexpr uint32_t kStOffBar = kStOffRed + 64;
constexpr uint32_t kStSmemBytes = kStOffBar + 64 + 1024;

// Review pooling folded into chunk_state (RUN > 0): along the scan's fastest axis the
// review box is RUN tokens long and RUN divides 128, so the rows of a sub-chunk come
// in runs of RUN consecutive rows that share one pooling cell. Warp w builds rows
// 32(w%4).. of the sub-chunk, columns 32g.. (g = w/4); its runs lie inside those rows,
// so each warp sums its own runs from the x tile before it scales the tile in place:
// a lane takes one (run, four columns) sum per RUN = 8 run, two per RUN = 4. The sums
// of x (this head), dt and, for the group's first head, B stay in registers while the
// lane's run in the next sub-chunk falls in the same cell (in time-major order the
// sub-chunks of a chunk are neighbouring rows of one box); when the cell changes they
// are added to the cell's totals with vector atomics. The separate pooling pass, which
// would read x, dt and B once more, is then not needed.
template <int RUN>
struct RunSums {
    static constexpr int NO = 8 / RUN;  // (run, four columns) sums per lane
    float x[NO][4], b[NO][4], d[NO];
    int cell[NO];  // -1: nothing held
};

// The lane's j-th run, counted in RUN-row runs from the warp's first row.
__device__ __forceinline__ int lane_run(int j) { return ((threadIdx.x & 31) >> 3) + 4 * j; }

// Adds to out the sums over the rows of the lane's runs of four bf16 columns
// (c4 = column / 4) of an SW128 tile. A warp reads rows of four runs at once; for RUN = 8 they alternate
// between the two halves of the swizzled row, so each read is two bank wavefronts.
template <int RUN>
__device__ __forceinline__ void run_sums(const uint8_t *tile, int rbase, int c4, float (&out)[8 / RUN][4])
{
#pragma unroll
    for (int j = 0; j < 8 / RUN; ++j) {
        const int rl = lane_run(j);
        float2 s01 = make_float2(out[j][0], out[j][1]), s23 = make_float2(out[j][2], out[j][3]);
#pragma unroll
        for (int i = 0; i < RUN; ++i) {  // packed fp32 pairs
            const int r = rbase + RUN * rl + (RUN == 8 ? (i ^ (4 * (rl & 1))) : i);
            const uint2 u = *reinterpret_cast<const uint2 *>(tile + tc::sw128(r, c4 >> 1) + (c4 & 1) * 8);
            s01 = tc::add_f32x2(s01, tc::unpack_bf16(u.x));
            s23 = tc::add_f32x2(s23, tc::unpack_bf16(u.y));
        }
        out[j][0] = s01.x, out[j][1] = s01.y, out[j][2] = s23.x, out[j][3] = s23.y;
    }
}

template <int RUN>
__device__ __forceinline__ void run_flush(const SsdArgs &a, const RunSums<RUN> &acc, int j, int h, int grp,
                                          int c4, bool with_d, bool with_b)
{
    if (acc.cell[j] < 0) return;
    float *cell = a.pooled + (size_t)acc.cell[j] * (a.nh * a.P + a.nh + a.G * a.Ns);
    atomicAdd(reinterpret_cast<float4 *>(cell + h * a.P + 4 * c4),
              make_float4(acc.x[j][0], acc.x[j][1], acc.x[j][2], acc.x[j][3]));
    if (with_d) atomicAdd(cell + a.nh * a.P + h, acc.d[j]);
    if (with_b)
        atomicAdd(reinterpret_cast<float4 *>(cell + a.nh * a.P + a.nh + grp * a.Ns + 4 * c4),
                  make_float4(acc.b[j][0], acc.b[j][1], acc.b[j][2], acc.b[j][3]));
}

template <int RUN>
__global__ void __launch_bounds__(kThreads, 4)
    ssd_chunk_state_tc_kernel(SsdArgs a, int nsub, const __grid_constant__ CUtensorMap mx,
                              const __grid_constant__ CUtensorMap mB, TmaRows geo)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t *tX = base + kStOffX, *tB = base + kStOffB, *ub = base + kStOffU;
    float *sdt = reinterpret_cast<float *>(base + kStOffDt);
    float *scum = reinterpret_cast<float *>(base + kStOffCum);
    int *sgoff = reinterpret_cast<int *>(base + kStOffGoff);
    float *sred = reinterpret_cast<float *>(base + kStOffRed);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + kStOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kStOffBar + 8);
    int *abort_flag = reinterpret_cast<int *>(base + kStOffBar + 12);
    uint64_t *ldbar = reinterpret_cast<uint64_t *>(base + kStOffBar + 16);  // TMA row loads

    const int tid = threadIdx.x, warp = tid >> 5;
    const int r = tid & (kSub - 1), g = tid >> 7;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
    const int h = blockIdx.x, c = blockIdx.y, b = blockIdx.z + geo.zbase;
    const int L = nsub * kSub;
    const int n0 = c * L, len = min(L, a.N - n0);
    const int grp = h / (a.nh / a.G);
    const float Ah = a.A[h];
    uint32_t mma_phase = 0, ld_issued = 0, ld_phase = 0;  // TMA batches issued / completed
    constexpr int RS = RUN > 0 ? RUN : 8;
    RunSums<RS> runs;
#pragma unroll
    for (int j = 0; j < RunSums<RS>::NO; ++j) runs.cell[j] = -1;
    const bool with_b = h % (a.nh / a.G) == 0;     // the group's first head pools B
    const bool with_d = g == 0 && (tid & 7) == 0;  // one lane per run pools dt
    const int c4 = 8 * g + (tid & 7), rbase = (warp & 3) * 32;

    if (warp == 0) tc::tmem_alloc(tmem_slot, 64);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(ldbar, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
        // TMA boxes need no grid offsets: sub-chunk 0's rows are requested first
        if (geo.use) tma_rows(&mx, &mB, nullptr, geo, tX, tB, nullptr, ldbar, h, grp, n0);
    }
    if (geo.use) ++ld_issued;
    load_chunk_meta(a, b, h, n0, len, L, sgoff, sdt);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // chunk_out loads this chunk's dt in scan order with one bulk copy
    {
        float4 *dst = reinterpret_cast<float4 *>(a.dt_scan + (((size_t)b * a.nh + h) * a.nchunks + c) * L);
        for (int i = tid; i < L / 4; i += kThreads) dst[i] = reinterpret_cast<const float4 *>(sdt)[i];
    }
    sub_cumsums(sdt, scum, Ah, nsub, true, sred);
    const float cend = scum[L - 1];

    for (int k = 0; k < nsub; ++k) {
        if (geo.use) {
            if (k > 0) {
                if (tid == 0) tma_rows(&mx, &mB, nullptr, geo, tX, tB, nullptr, ldbar, h, grp, n0 + k * kSub);
                ++ld_issued;
            }
            if (tc::mbar_wait(ldbar, ld_phase & 1u, a.err))
                ++ld_phase;
            else
                *abort_flag = 1;
        } else {
            load_rows(a, tX, tB, nullptr, sgoff, b, h, grp, len, k);
            wait_loads(false);
        }
        __syncthreads();
        if (*abort_flag) goto done;
        if constexpr (RUN > 0) {
            // this warp's runs of the unscaled x; a run's cell from its first row's grid position
#pragma unroll
            for (int j = 0; j < RunSums<RUN>::NO; ++j) {
                const int n0r = k * kSub + rbase + RUN * lane_run(j);
                int cell = -1;
                if (n0r < len) {
                    const uint32_t gg = (uint32_t)sgoff[n0r];
                    const uint32_t t = fdiv(gg, a.dHW), rem = gg - t * a.dHW.d;
                    const uint32_t hh = fdiv(rem, a.dW), ww = rem - hh * a.dW.d;
                    cell = b * a.Np + (int)((fdiv(t, a.dpt) * a.Hp + fdiv(hh, a.dph)) * a.Wp + fdiv(ww, a.dpw));
                }
                if (cell != runs.cell[j]) {
                    run_flush<RUN>(a, runs, j, h, grp, c4, with_d, with_b);
                    runs.cell[j] = cell;
                    runs.d[j] = 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) runs.x[j][e] = runs.b[j][e] = 0.f;
                }
            }
            run_sums<RUN>(tX, rbase, c4, runs.x);
            __syncwarp();  // the reads above come before this warp's in-place scaling
        }
        {
            const int n = k * kSub + r;
            const float cj = scum[n], dj = sdt[n];
            uint4 xv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[q] = *reinterpret_cast<const uint4 *>(tX + tc::sw128(r, 4 * g + q));
            const __nv_bfloat162 f2 = __float2bfloat162_rn(__expf(cend - cj) * dj);
            const __nv_bfloat162 b2 = __float2bfloat162_rn(__expf(cj - dj * Ah) * dj);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = tc::sw128(r, 4 * g + q);
                *reinterpret_cast<uint4 *>(tX + off) = scale_chunk(xv[q], f2);
                *reinterpret_cast<uint4 *>(ub + off) = scale_chunk(xv[q], b2);
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            mma_states(tmem, tc::smem_u32(tX), tc::smem_u32(tB), k > 0);
            tc::mma_commit(bar);
        }
        if constexpr (RUN > 0) {
            // while the MMA runs: the runs' sums of dt and of B (which the MMA only reads)
#pragma unroll
            for (int j = 0; j < RunSums<RUN>::NO; ++j) {
                if (with_d) {
                    const float *d = sdt + k * kSub + rbase + RUN * lane_run(j);
                    float sd = 0.f;
#pragma unroll
                    for (int i = 0; i < RUN; ++i) sd += d[i];
                    runs.d[j] += sd;
                }
            }
            if (with_b) run_sums<RUN>(tB, rbase, c4, runs.b);
        }
        if (!mma_wait(bar, mma_phase, a.err, abort_flag)) goto done;
    }
    {
        // TMEM rows 0-63: forward state rows p, rows 64-127: flipped state rows p (stored as bf16)
        const bool fwd = r < 64;
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(fwd ? a.states_f : a.states_b) +
                             ((((size_t)b * a.nh + h) * a.nchunks + c) * 64 + (r & 63)) * 64 + 32 * g;
        float v[32];
        tc::tmem_ld32(tc::tmem_addr(tmem, lane_base, 32 * g), v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = tc::pack_bf16(v[8 * q], v[8 * q + 1]);
            o.y = tc::pack_bf16(v[8 * q + 2], v[8 * q + 3]);
            o.z = tc::pack_bf16(v[8 * q + 4], v[8 * q + 5]);
            o.w = tc::pack_bf16(v[8 * q + 6], v[8 * q + 7]);
            *reinterpret_cast<uint4 *>(dst + 8 * q) = o;
        }
        if (tid == 0) a.alpha[((size_t)b * a.nh + h) * a.nchunks + c] = __expf(cend);
        if constexpr (RUN > 0) {
#pragma unroll
            for (int j = 0; j < RunSums<RUN>::NO; ++j) run_flush<RUN>(a, runs, j, h, grp, c4, with_d, with_b);
        }
    }
done:
    tc::cp_async_wait_all();
    // after a timeout a TMA batch may still be landing: a second bounded wait for it
    if (ld_issued > ld_phase && tid == 0) tc::mbar_wait(ldbar, ld_phase & 1u, nullptr);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 64);
    }
}

// ---------------------------------------------------------------------------
// state_chain: one thread per eight consecutive elements of the 64 x 64 state
// (one 16-byte vector). The chunk states are stored as bf16; the chain itself
// runs in fp32, with the loads of kAhead chunks in flight ahead of it. Three CTAs
// per SM, so that the 320 CTAs of an 80-head grid all run at once (no tail wave).
// grid: (4096 / 8 / kChainThreads, nh * batch, 2 directions)
// ---------------------------------------------------------------------------
constexpr int kAhead = 8;
constexpr int kChainThreads = 256;

__global__ void __launch_bounds__(kChainThreads, 3) ssd_state_chain_kernel(SsdArgs a)
{
    const int e8 = (blockIdx.x * kChainThreads + threadIdx.x) * 8;  // first of this thread's 8 elements
    const int hb = blockIdx.y, dir = blockIdx.z;
    const int h = hb % a.nh, b = hb / a.nh;
    const int nc = a.nchunks;
    __nv_bfloat16 *S = reinterpret_cast<__nv_bfloat16 *>(dir == 0 ? a.states_f : a.states_b) +
                       ((size_t)b * a.nh + h) * nc * 4096 + e8;
    const float *al = a.alpha + ((size_t)b * a.nh + h) * nc;
    float hv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) hv[j] = 0.f;
    if (a.review) {  // h_init comes in parts over ranges of review cells
        for (int part = 0; part < kHinitParts; ++part) {
            const float4 *src = reinterpret_cast<const float4 *>(
                a.h_init + (((size_t)part * a.batch + b) * a.nh + h) * 4096 + e8);
            const float4 u = src[0], v = src[1];
            hv[0] += u.x, hv[1] += u.y, hv[2] += u.z, hv[3] += u.w;
            hv[4] += v.x, hv[5] += v.y, hv[6] += v.z, hv[7] += v.w;
        }
    }
    // one chain step: the stored chunk-local state becomes the entering state
    auto step_chunk = [&](int cidx, uint4 loc, float alpha) {
        uint4 o;
        o.x = tc::pack_bf16(hv[0], hv[1]);
        o.y = tc::pack_bf16(hv[2], hv[3]);
        o.z = tc::pack_bf16(hv[4], hv[5]);
        o.w = tc::pack_bf16(hv[6], hv[7]);
        *reinterpret_cast<uint4 *>(S + (size_t)cidx * 4096) = o;
        const uint32_t w4[4] = {loc.x, loc.y, loc.z, loc.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 hn = tc::fma_f32x2(make_float2(alpha, alpha), make_float2(hv[2 * q], hv[2 * q + 1]),
                                            tc::unpack_bf16(w4[q]));
            hv[2 * q] = hn.x, hv[2 * q + 1] = hn.y;
        }
    };
    // visit chunks in chain order: forward 0 .. nc-1, flipped nc-1 .. 0
    const int step = dir == 0 ? 1 : -1;
    int cidx = dir == 0 ? 0 : nc - 1;
    int left = nc;
    while (left >= kAhead) {
        uint4 buf[kAhead];
        float alp[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            buf[u] = *reinterpret_cast<const uint4 *>(S + (size_t)(cidx + u * step) * 4096);
            alp[u] = al[cidx + u * step];
        }
#pragma unroll
        for (int u = 0; u < kAhead; ++u) step_chunk(cidx + u * step, buf[u], alp[u]);
        cidx += kAhead * step;
        left -= kAhead;
    }
    for (; left > 0; --left, cidx += step)
        step_chunk(cidx, *reinterpret_cast<const uint4 *>(S + (size_t)cidx * 4096), al[cidx]);
}

}  // namespace

bool ssd_tc_supported(const SsdArgs &a)
{
    return a.bf16 && a.P == 64 && a.Ns == 64 && a.dirs == MATE_DIR_BI && a.Q % kSub == 0 && a.Q / kSub >= 1 &&
           a.Q / kSub <= kMaxSubs && a.nchunks <= 65535 && a.nh <= 65535 && a.batch <= 65535 &&
           (size_t)a.nh * a.batch <= 65535;
}

cudaError_t launch_ssd_tc(const SsdArgs &a, cudaStream_t s)
{
    cudaError_t e = cudaFuncSetAttribute(ssd_chunk_out_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    // the review pooling folds into chunk_state when the review box is 4 or 8 tokens
    // long along the scan's fastest axis and the channel blocks allow 16-byte atomics
    int run = 0;
    if (a.review) {
        // (the zigzag scan walks W inside each row, either way: runs of pw along W)
        const int r0 = (a.mode == MATE_SCAN_SR || a.mode == MATE_SCAN_ZZ) ? a.pw
                       : (a.mode == MATE_SCAN_SC ? a.ph : a.pt);
        if ((r0 == 4 || r0 == 8) && a.nh % 4 == 0 && (a.G * a.Ns) % 4 == 0) run = r0;
    }
    auto st_kernel = run == 8 ? ssd_chunk_state_tc_kernel<8>
                              : (run == 4 ? ssd_chunk_state_tc_kernel<4> : ssd_chunk_state_tc_kernel<0>);
    e = cudaFuncSetAttribute(st_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStSmemBytes);
    if (e != cudaSuccess) return e;
    SsdArgs ar = a;  // the review scan reads one part of the box sums when they are pooled here
    if (a.review) {
        if (run) {
            ar.pool_splits = 1;
            Phase ph(MATE_PHASE_REVIEW_POOL, s);
            e = cudaMemsetAsync(a.pooled, 0,
                                (size_t)a.batch * a.Np * ((size_t)a.nh * a.P + a.nh + (size_t)a.G * a.Ns) * 4, s);
        } else {
            e = launch_review_pool_bf16_64(a, s);
        }
        if (e != cudaSuccess) return e;
    }
    const int nsub = a.Q / kSub;
    // TMA row boxes when the scan order allows them: one launch per batch element
    struct Maps {
        CUtensorMap x, b, c, o;
    };
    const ScanBox sb = scan_box(a.mode, a.T, a.H, a.W);
    auto build_maps = [&](int bb, Maps &m) {
        const uint64_t tx = (uint64_t)a.nh * 64 * 2, tb = (uint64_t)a.G * 64 * 2;  // token strides in bytes
        const uint64_t dx[5] = {64, (uint64_t)a.nh, (uint64_t)sb.n[0], (uint64_t)sb.n[1], (uint64_t)sb.n[2]};
        const uint64_t db[5] = {64, (uint64_t)a.G, (uint64_t)sb.n[0], (uint64_t)sb.n[1], (uint64_t)sb.n[2]};
        const uint64_t sx[4] = {128, sb.stride[0] * tx, sb.stride[1] * tx, sb.stride[2] * tx};
        const uint64_t sbs[4] = {128, sb.stride[0] * tb, sb.stride[1] * tb, sb.stride[2] * tb};
        const uint32_t box[5] = {64, 1, sb.box[0], sb.box[1], sb.box[2]};
        const size_t tok = (size_t)bb * a.N;
        return tmap_bf16_5d(&m.x, static_cast<const __nv_bfloat16 *>(a.x) + tok * a.nh * 64, dx, sx, box) &&
               tmap_bf16_5d(&m.b, static_cast<const __nv_bfloat16 *>(a.B) + tok * a.G * 64, db, sbs, box) &&
               tmap_bf16_5d(&m.c, static_cast<const __nv_bfloat16 *>(a.C) + tok * a.G * 64, db, sbs, box) &&
               tmap_bf16_5d(&m.o, static_cast<const __nv_bfloat16 *>(a.out) + tok * a.nh * 64, dx, sx, box);
    };
    Maps maps = {};
    TmaRows geo = {0, 1, 1, 0};
    if (sb.ok && tmap_available() && build_maps(0, maps)) {
        geo.use = 1;
        geo.n0 = sb.n[0];
        geo.n1 = sb.n[1];
    }
    const int launches = geo.use ? a.batch : 1, zdim = geo.use ? 1 : a.batch;
    for (int l = 0; l < launches; ++l) {
        if (geo.use && !build_maps(l, maps)) return cudaErrorInvalidValue;
        geo.zbase = geo.use ? l : 0;
        Phase ph(MATE_PHASE_CHUNK_STATE, s);
        st_kernel<<<dim3(a.nh, a.nchunks, zdim), kThreads, kStSmemBytes, s>>>(a, nsub, maps.x, maps.b, geo);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.review) {
        e = launch_review_scan_bf16_64(ar, s);
        if (e != cudaSuccess) return e;
    }
    {
        Phase ph(MATE_PHASE_STATE_PASS, s);
        ssd_state_chain_kernel<<<dim3(4096 / 8 / kChainThreads, a.nh * a.batch, 2), kChainThreads, 0, s>>>(a);
    }
    // chunk_out is persistent: two CTAs per SM walk the (head, chunk, batch) items
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int nitems = a.nh * a.nchunks * zdim;
    const int grid = std::min(nitems, 2 * std::max(nsm, 1));
    for (int l = 0; l < launches; ++l) {
        if (geo.use && !build_maps(l, maps)) return cudaErrorInvalidValue;
        geo.zbase = geo.use ? l : 0;
        Phase ph(MATE_PHASE_CHUNK_OUT, s);
        ssd_chunk_out_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a, nsub, maps.x, maps.b, maps.c, maps.o, geo,
                                                                  nitems);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace mate
