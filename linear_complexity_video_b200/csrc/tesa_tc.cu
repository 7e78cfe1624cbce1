// TEmporal Swin Attention on the 5th-generation tensor cores (tcgen05, TMEM,
// TMA) for bf16 storage, head dim 128 and 128-token windows (Tw*Sw*Sw = 128).
//
// Method (paper review "LinGen ...", section 三, TE-Branch): each token
// attends to the tokens of its own Tw x Sw x Sw window; the window grid is
// shifted on alternate layers, with partial windows at both ends of a shifted
// axis.
//
// One CTA of 128 threads per (window, head); two CTAs fit on an SM (96 KB of
// shared memory and 256 TMEM columns each), so one CTA's loads overlap the
// other's math.
//   1. TMA loads the window's Q, K, V boxes (64 head-dims x Sw x Sw x Tw each,
//      two per tensor) straight from the (T, H, W, heads, d) layout. The box
//      origin is the window's first grid coordinate, possibly negative for a
//      shifted window; TMA fills out-of-grid rows with zeros. The shift lives
//      entirely in these coordinates.
//   2. S = Q K^T (M = N = K = 128) into TMEM.
//   3. Thread i owns query i: it reads S row i from TMEM, masks keys outside
//      the grid, and writes P = exp(S - max) as bf16 into shared memory
//      (reusing Q's buffer) in the swizzled K-major operand layout.
//   4. O = P V (V as an MN-major operand) into TMEM.
//   5. Thread i scales O row i by 1 / sum(P) and stores it if query i is in
//      the grid.
// A window holds exactly one 128-token tile, so the softmax needs no online
// rescaling.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace mate {

namespace {

constexpr int kThreads = 128;
constexpr uint32_t kTile = 16384;  // one 128-row x 128-byte box
constexpr uint32_t kSmemData = 6 * kTile;
constexpr uint32_t kSmemBytes = kSmemData + 1024 /*alignment slack*/ + 64;  // + barriers, flags, key mask

struct TesaTcParams {
    int T, H, W, nh;
    int Tw, Sw;
    int offt, offh, offw;
    int nwh, nww;
    float scale_log2;   // log2(e) / sqrt(d)
    __nv_bfloat16 *out; // batch element base
    int *err;
};

__global__ void __launch_bounds__(kThreads, 2)
    tesa_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, TesaTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t *sQ = smem;              // 2 tiles; later holds P
    uint8_t *sK = smem + 2 * kTile;  // 2 tiles
    uint8_t *sV = smem + 4 * kTile;  // 2 tiles
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(smem + kSmemData);
    uint64_t *bar_mma = bar_load + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int head = blockIdx.x, wid = blockIdx.y;  // heads fastest: they share DRAM rows
    const int kw = wid % p.nww, kh = (wid / p.nww) % p.nwh, kt = wid / (p.nww * p.nwh);
    const int t0 = kt * p.Tw - p.offt, h0 = kh * p.Sw - p.offh, w0 = kw * p.Sw - p.offw;

    if (warp == 0) tc::tmem_alloc(tmem_slot, 256);
    if (tid == 0) {
        tc::mbar_init(bar_load, 1);
        tc::mbar_init(bar_mma, 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;

    if (tid == 0) {
        tc::mbar_expect_tx(bar_load, 6 * kTile);
        for (int half = 0; half < 2; ++half) {
            tc::tma_load_5d(sQ + half * kTile, &mq, bar_load, half * 64, head, w0, h0, t0);
            tc::tma_load_5d(sK + half * kTile, &mk, bar_load, half * 64, head, w0, h0, t0);
            tc::tma_load_5d(sV + half * kTile, &mv, bar_load, half * 64, head, w0, h0, t0);
        }
    }

    // which of the 128 box rows are inside the grid (row r = (tt*Sw + hh)*Sw + ww)
    const int ss = p.Sw * p.Sw;
    auto row_valid = [&](int r) {
        const int tt = t0 + r / ss, hh = h0 + (r / p.Sw) % p.Sw, ww = w0 + r % p.Sw;
        return tt >= 0 && tt < p.T && hh >= 0 && hh < p.H && ww >= 0 && ww < p.W;
    };
    // key validity mask: thread r evaluates row r once, warp ballots share it
    uint32_t *smask = reinterpret_cast<uint32_t *>(abort_flag + 1);
    const bool qvalid = row_valid(tid);
    {
        const uint32_t m = __ballot_sync(0xffffffffu, qvalid);
        if ((tid & 31) == 0) smask[warp] = m;
    }

    if (!tc::mbar_wait(bar_load, 0, p.err)) atomicExch(abort_flag, 1);
    __syncthreads();
    if (*abort_flag) {
        tc::mbar_wait(bar_load, 0, nullptr);  // bounded second chance for copies in flight
        goto cleanup;
    }
    uint32_t kmask[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) kmask[c] = smask[c];

    // ---- S = Q K^T --------------------------------------------------------
    if (tid == 0) {
        tc::tc_fence_after();
        const uint32_t idesc = tc::idesc_bf16(128, 128, 0, 0);
        const uint32_t q0 = tc::smem_u32(sQ), k0 = tc::smem_u32(sK);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s >> 2) * kTile + (s & 3) * 32;
            tc::mma_bf16(tS, tc::sdesc_sw128(q0 + off, 16, 1024), tc::sdesc_sw128(k0 + off, 16, 1024), idesc, s > 0);
        }
        tc::mma_commit(bar_mma);
    }
    if (!tc::mbar_wait(bar_mma, 0, p.err)) atomicExch(abort_flag, 1);
    __syncthreads();
    if (*abort_flag) {
        tc::mbar_wait(bar_mma, 0, nullptr);
        goto cleanup;
    }
    tc::tc_fence_after();

    // ---- softmax of row tid -> P (bf16, K-major swizzled, into sQ) ---------
    {
        const uint32_t lane_base = (uint32_t)(warp * 32);
        float s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld32(tc::tmem_addr(tS, lane_base, c * 32), s[c]);
        tc::tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if ((kmask[c] >> j) & 1u) mx = fmaxf(mx, s[c][j]);
        const float mxs = mx * p.scale_log2;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float e = ((kmask[c] >> j) & 1u) ? exp2f(fmaf(s[c][j], p.scale_log2, -mxs)) : 0.f;
                s[c][j] = e;
                sum += e;
            }
        // row tid of P: keys 0..63 in tile 0, 64..127 in tile 1; 8 keys per 16-byte chunk
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int key0 = c * 32 + q * 8;
                uint4 v;
                v.x = tc::pack_bf16(s[c][q * 8 + 0], s[c][q * 8 + 1]);
                v.y = tc::pack_bf16(s[c][q * 8 + 2], s[c][q * 8 + 3]);
                v.z = tc::pack_bf16(s[c][q * 8 + 4], s[c][q * 8 + 5]);
                v.w = tc::pack_bf16(s[c][q * 8 + 6], s[c][q * 8 + 7]);
                uint8_t *tile = sQ + (key0 >> 6) * kTile;
                *reinterpret_cast<uint4 *>(tile + tc::sw128(tid, (key0 & 63) >> 3)) = v;
            }
        const float inv = 1.f / sum;
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ---- O = P V ---------------------------------------------------------
        if (tid == 0) {
            tc::tc_fence_after();
            const uint32_t idesc = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t p0 = tc::smem_u32(sQ), v0 = tc::smem_u32(sV);
#pragma unroll
            for (int st = 0; st < 8; ++st) {
                const uint32_t aoff = (st >> 2) * kTile + (st & 3) * 32;
                tc::mma_bf16(tO, tc::sdesc_sw128(p0 + aoff, 16, 1024), tc::sdesc_sw128(v0 + st * 2048, kTile, 1024),
                             idesc, st > 0);
            }
            tc::mma_commit(bar_mma);
        }
        if (!tc::mbar_wait(bar_mma, 1, p.err)) atomicExch(abort_flag, 1);
        __syncthreads();
        if (*abort_flag) {
            tc::mbar_wait(bar_mma, 1, nullptr);
            goto cleanup;
        }
        tc::tc_fence_after();

        // ---- epilogue: row tid of O / sum -> global --------------------------
        const int tt = t0 + tid / ss, hh = h0 + (tid / p.Sw) % p.Sw, ww = w0 + tid % p.Sw;
        __nv_bfloat16 *dst =
            qvalid ? p.out + ((((size_t)tt * p.H + hh) * p.W + ww) * p.nh + head) * 128 : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float o[32];
            tc::tmem_ld32(tc::tmem_addr(tO, lane_base, c * 32), o);
            tc::tmem_wait_ld();
            if (qvalid) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 v;
                    v.x = tc::pack_bf16(o[q * 8 + 0] * inv, o[q * 8 + 1] * inv);
                    v.y = tc::pack_bf16(o[q * 8 + 2] * inv, o[q * 8 + 3] * inv);
                    v.z = tc::pack_bf16(o[q * 8 + 4] * inv, o[q * 8 + 5] * inv);
                    v.w = tc::pack_bf16(o[q * 8 + 6] * inv, o[q * 8 + 7] * inv);
                    *reinterpret_cast<uint4 *>(dst + c * 32 + q * 8) = v;
                }
            }
        }
    }

cleanup:
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// (batch element of a (T, H, W, nh, 128) bf16 tensor) -> 5-D map, box = 64 x 1 x Sw x Sw x Tw
bool make_map(CUtensorMap *m, const void *base, const TesaArgs &a)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t e = 2;
    cuuint64_t dims[5] = {128, (cuuint64_t)a.nh, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.T};
    cuuint64_t strides[4] = {128 * e, (cuuint64_t)a.nh * 128 * e, (cuuint64_t)a.W * a.nh * 128 * e,
                             (cuuint64_t)a.H * a.W * a.nh * 128 * e};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)a.Sw, (cuuint32_t)a.Sw, (cuuint32_t)a.Tw};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool tesa_tc_supported(const TesaArgs &a)
{
    return a.bf16 && a.d == 128 && a.Tw * a.Sw * a.Sw == 128 && a.Sw <= 128 && a.Tw <= 128 &&
           (size_t)a.nwt * a.nwh * a.nww <= 65535 &&
           encode_fn() != nullptr;
}

cudaError_t launch_tesa_tc(const TesaArgs &a, cudaStream_t s)
{
    cudaError_t e = cudaFuncSetAttribute(tesa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    TesaTcParams p;
    p.T = a.T;
    p.H = a.H;
    p.W = a.W;
    p.nh = a.nh;
    p.Tw = a.Tw;
    p.Sw = a.Sw;
    p.offt = a.offt;
    p.offh = a.offh;
    p.offw = a.offw;
    p.nwh = a.nwh;
    p.nww = a.nww;
    p.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
    p.err = a.err;
    const size_t per_batch = (size_t)a.N * a.nh * 128;
    const int nwin = a.nwt * a.nwh * a.nww;
    for (int b = 0; b < a.batch; ++b) {
        CUtensorMap mq, mk, mv;
        const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q) + b * per_batch;
        const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(a.k) + b * per_batch;
        const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(a.v) + b * per_batch;
        if (!make_map(&mq, q, a) || !make_map(&mk, k, a) || !make_map(&mv, v, a)) return cudaErrorInvalidValue;
        p.out = static_cast<__nv_bfloat16 *>(a.out) + b * per_batch;
        Phase ph(MATE_PHASE_TESA, s);
        tesa_tc_kernel<<<dim3(a.nh, nwin), kThreads, kSmemBytes, s>>>(mq, mk, mv, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mate
