// TEmporal Swin Attention on the 5th-generation tensor cores (tcgen05, TMEM,
// TMA) for bf16 storage, head dim 128 and 128-token windows (Tw*Sw*Sw = 128).
//
// Method (paper review "LinGen ...", section 三, TE-Branch): each token
// attends to the tokens of its own Tw x Sw x Sw window; the window grid is
// shifted on alternate layers, with partial windows at both ends of a shifted
// axis.
//
// One persistent CTA per SM walks (window, head) items with two shared-memory
// stages and two TMEM buffers, so the loads of one item, the tensor-core work
// of another and the softmax of a third overlap: a producer warp issues the
// TMA loads, an MMA warp issues tcgen05.mma, and two warpgroups take turns
// with the softmax and the epilogue.
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

constexpr uint32_t kTile = 16384;           // one 128-row x 128-byte box
constexpr uint32_t kStage = 6 * kTile;      // Q (2 tiles, later P), K (2), V (2)
constexpr int kStages = 2;
constexpr int kWG = 128;                    // a softmax / epilogue warpgroup
constexpr int kProducerWarp = 8;            // TMA loads
constexpr int kMmaWarp = 9;                 // tcgen05.mma issue
constexpr int kThreads = 320;               // warpgroups 0 and 1 (warps 0-7), producer, MMA
constexpr uint32_t kSmemBytes = kStages * kStage + 1024 /*alignment slack*/ + 256;

struct TesaTcParams {
    int T, H, W, nh;
    int Tw, Sw;
    int offt, offh, offw;
    int nwh, nww;
    int items;          // windows * heads
    float scale_log2;   // log2(e) / sqrt(d)
    __nv_bfloat16 *out; // batch element base
    int *err;
};

struct Item {
    int head, t0, h0, w0;
};

// Items are ordered (window, head) with heads fastest and dealt round-robin:
// CTA c takes c, c + G, c + 2G, ... (G CTAs), so at any moment the CTAs work
// on neighbouring windows and share DRAM rows and L2 lines.
__device__ __forceinline__ Item item_of(const TesaTcParams &p, int local)
{
    const int item = blockIdx.x + local * gridDim.x;
    Item it;
    it.head = item % p.nh;
    const int wid = item / p.nh;
    const int kw = wid % p.nww, kh = (wid / p.nww) % p.nwh, kt = wid / (p.nww * p.nwh);
    it.t0 = kt * p.Tw - p.offt;
    it.h0 = kh * p.Sw - p.offh;
    it.w0 = kw * p.Sw - p.offw;
    return it;
}

// is box row r (r = (tt*Sw + hh)*Sw + ww) inside the grid?
__device__ __forceinline__ bool row_in_grid(const TesaTcParams &p, const Item &it, int r)
{
    const int ss = p.Sw * p.Sw;
    const int tt = it.t0 + r / ss, hh = it.h0 + (r / p.Sw) % p.Sw, ww = it.w0 + r % p.Sw;
    return tt >= 0 && tt < p.T && hh >= 0 && hh < p.H && ww >= 0 && ww < p.W;
}

// Persistent CTA (one per SM) walking its share of the items; its i-th item
// uses smem stage i % 2 and TMEM buffers S[i % 2], O[i % 2].
//   producer warp : TMA Q, K, V of item i into its stage once the stage is free
//   MMA warp      : S = Q K^T once loaded (and the TMEM buffer is free);
//                   O = P V once the warpgroup has written P
//   warpgroups    : warpgroup g takes the items with i % 2 == g: softmax into
//                   P, then (after P V) the epilogue
__global__ void __launch_bounds__(kThreads, 1)
    tesa_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, TesaTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * kStage);
    uint64_t *full = bars;         // [2] stage loaded
    uint64_t *empty = bars + 2;    // [2] stage consumed (P V done)
    uint64_t *s_full = bars + 4;   // [2] S in TMEM
    uint64_t *p_full = bars + 6;   // [2] P written (128 arrivals)
    uint64_t *o_full = bars + 8;   // [2] O in TMEM
    uint64_t *t_empty = bars + 10; // [2] O read out (128 arrivals)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 12);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_items = p.items > (int)blockIdx.x ? (p.items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
            tc::mbar_init(&s_full[i], 1);
            tc::mbar_init(&p_full[i], kWG);
            tc::mbar_init(&o_full[i], 1);
            tc::mbar_init(&t_empty[i], kWG);
        }
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Waits inside a role are made warp-uniform, so a warp leaves its loop as a
    // whole and every thread reaches the final __syncthreads.
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, tc::mbar_wait_or_abort(bar, parity, p.err, abort_flag)) != 0;
    };
    if (warp == kProducerWarp) {
        for (int i = 0; i < n_items; ++i) {
            const int s = i & 1;
            if (i >= 2 && !wait_all(&empty[s], ((i >> 1) - 1) & 1)) break;
            if (lane == 0) {
                const Item it = item_of(p, i);
                uint8_t *st = smem + s * kStage;
                tc::mbar_expect_tx(&full[s], kStage);
                for (int half = 0; half < 2; ++half) {
                    tc::tma_load_5d(st + half * kTile, &mq, &full[s], half * 64, it.head, it.w0, it.h0, it.t0);
                    tc::tma_load_5d(st + (2 + half) * kTile, &mk, &full[s], half * 64, it.head, it.w0, it.h0, it.t0);
                    tc::tma_load_5d(st + (4 + half) * kTile, &mv, &full[s], half * 64, it.head, it.w0, it.h0, it.t0);
                }
            }
            __syncwarp();
        }
    } else if (warp == kMmaWarp) {
        // S(i+1) is issued before waiting for P(i), so both warpgroups stay busy
        const uint32_t id_s = tc::idesc_bf16(128, 128, 0, 0);
        const uint32_t id_o = tc::idesc_bf16(128, 128, 0, 1);
        auto issue_s = [&](int i) -> bool {
            const int s = i & 1;
            const uint32_t ph = (i >> 1) & 1;
            if (!wait_all(&full[s], ph)) return false;
            if (i >= 2 && !wait_all(&t_empty[s], ph ^ 1)) return false;
            tc::tc_fence_after();
            if (lane == 0) {
                const uint32_t q0 = tc::smem_u32(smem + s * kStage), k0 = q0 + 2 * kTile;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * kTile + (k & 3) * 32;
                    tc::mma_bf16(tmem + s * 256, tc::sdesc_sw128(q0 + off, 16, 1024), tc::sdesc_sw128(k0 + off, 16, 1024),
                                 id_s, k > 0);
                }
                tc::mma_commit(&s_full[s]);
            }
            __syncwarp();
            return true;
        };
        if (n_items > 0 && issue_s(0)) {
            for (int i = 0; i < n_items; ++i) {
                if (i + 1 < n_items && !issue_s(i + 1)) break;
                const int s = i & 1;
                if (!wait_all(&p_full[s], (i >> 1) & 1)) break;
                tc::tc_fence_after();
                if (lane == 0) {
                    const uint32_t p0 = tc::smem_u32(smem + s * kStage), v0 = p0 + 4 * kTile;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t aoff = (k >> 2) * kTile + (k & 3) * 32;
                        tc::mma_bf16(tmem + s * 256 + 128, tc::sdesc_sw128(p0 + aoff, 16, 1024),
                                     tc::sdesc_sw128(v0 + k * 2048, kTile, 1024), id_o, k > 0);
                    }
                    tc::mma_commit(&o_full[s]);
                    tc::mma_commit(&empty[s]);
                }
                __syncwarp();
            }
        }
    } else {
        // ---- warpgroup g handles the items i with i % 2 == g (stage and TMEM buffer g)
        const int g = warp >> 2, row = tid & (kWG - 1);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const uint32_t tS = tmem + g * 256, tO = tS + 128;
        for (int i = g; i < n_items; i += 2) {
            const uint32_t ph = (i >> 1) & 1;
            const Item it = item_of(p, i);
            // key validity: each warp ballots all 128 rows itself
            uint32_t kmask[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) kmask[c] = __ballot_sync(0xffffffffu, row_in_grid(p, it, c * 32 + lane));
            if (!wait_all(&s_full[g], ph)) break;
            tc::tc_fence_after();
            // pass 1: row maximum over the keys in the grid
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float sv[32];
                tc::tmem_ld32(tc::tmem_addr(tS, lane_base, c * 32), sv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if ((kmask[c] >> j) & 1u) mx = fmaxf(mx, sv[j]);
            }
            // pass 2: P = exp(S - max) as bf16 into the stage's Q tiles, and the row sum
            const float mxs = mx * p.scale_log2;
            float sum = 0.f;
            uint8_t *pq = smem + g * kStage;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float sv[32];
                tc::tmem_ld32(tc::tmem_addr(tS, lane_base, c * 32), sv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float e = ((kmask[c] >> j) & 1u) ? exp2f(fmaf(sv[j], p.scale_log2, -mxs)) : 0.f;
                    sv[j] = e;
                    sum += e;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key0 = c * 32 + q * 8;
                    uint4 v;
                    v.x = tc::pack_bf16(sv[q * 8 + 0], sv[q * 8 + 1]);
                    v.y = tc::pack_bf16(sv[q * 8 + 2], sv[q * 8 + 3]);
                    v.z = tc::pack_bf16(sv[q * 8 + 4], sv[q * 8 + 5]);
                    v.w = tc::pack_bf16(sv[q * 8 + 6], sv[q * 8 + 7]);
                    *reinterpret_cast<uint4 *>(pq + (key0 >> 6) * kTile + tc::sw128(row, (key0 & 63) >> 3)) = v;
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(&p_full[g]);
            const float inv = 1.f / sum;

            // epilogue: O row / sum -> global, once P V is done
            if (!wait_all(&o_full[g], ph)) break;
            tc::tc_fence_after();
            const bool qvalid = row_in_grid(p, it, row);
            const int ss = p.Sw * p.Sw;
            const int tt = it.t0 + row / ss, hh = it.h0 + (row / p.Sw) % p.Sw, ww = it.w0 + row % p.Sw;
            __nv_bfloat16 *dst =
                qvalid ? p.out + ((((size_t)tt * p.H + hh) * p.W + ww) * p.nh + it.head) * 128 : nullptr;
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
            tc::tc_fence_before();
            tc::mbar_arrive(&t_empty[g]);
        }
    }

    // all roles done (or aborted): make sure no MMA still writes TMEM, then free it
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // an aborted pipeline may still have copies or MMAs in flight: give them a
        // bounded 200 us to land before the tensor memory is released
        const uint64_t t0 = tc::globaltimer();
        while (tc::globaltimer() - t0 < 200000ull) {
        }
    }
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
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
           (size_t)a.nwt * a.nwh * a.nww * a.nh < ((size_t)1 << 31) &&
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
    p.items = nwin * a.nh;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = p.items < sms ? p.items : sms;
    for (int b = 0; b < a.batch; ++b) {
        CUtensorMap mq, mk, mv;
        const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q) + b * per_batch;
        const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(a.k) + b * per_batch;
        const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(a.v) + b * per_batch;
        if (!make_map(&mq, q, a) || !make_map(&mk, k, a) || !make_map(&mv, v, a)) return cudaErrorInvalidValue;
        p.out = static_cast<__nv_bfloat16 *>(a.out) + b * per_batch;
        Phase ph(MATE_PHASE_TESA, s);
        tesa_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mate
