// TEmporal Swin Attention on the 5th-generation tensor cores (tcgen05, TMEM,
// TMA) for bf16 storage, head dim 128 and 128-token windows (Tw*Sw*Sw = 128).
//
// Method (paper review "LinGen ...", section 三, TE-Branch): each token
// attends to the tokens of its own Tw x Sw x Sw window; the window grid is
// shifted on alternate layers, with partial windows at both ends of a shifted
// axis.
//
// One persistent CTA per SM walks (window, head) items. Q and K of an item sit
// in one of two shared-memory slots that are released as soon as S = Q K^T is
// done; V sits in one of two slots released after O = P V; P goes to TMEM
// over S (the A operand of P V is read from TMEM). Two warps issue the TMA
// loads (Q+K and V), one warp issues tcgen05.mma, and two warpgroups take
// turns with the softmax and the epilogue, so loads, tensor-core work and
// softmax of neighbouring items overlap.
//   1. TMA loads the window's Q, K, V boxes (64 head-dims x Sw x Sw x Tw each,
//      two per tensor) straight from the (T, H, W, heads, d) layout. The box
//      origin is the window's first grid coordinate, possibly negative for a
//      shifted window; TMA fills out-of-grid rows with zeros. The shift lives
//      entirely in these coordinates.
//   2. S = Q K^T (M = N = K = 128) into TMEM.
//   3. Thread i owns query i: it reads S row i from TMEM, masks keys outside
//      the grid, and writes P = exp(S - max) as bf16 pairs back into TMEM.
//   4. O = P V (P from TMEM, V as an MN-major shared-memory operand) into TMEM.
//   5. Thread i scales O row i by 1 / sum(P); each warp stages its 32 rows in
//      shared memory and stores those of queries in the grid as whole lines.
// A window holds exactly one 128-token tile, so the softmax needs no online
// rescaling.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace mate {

namespace {

constexpr uint32_t kTile = 16384;           // one 128-row x 128-byte box
constexpr int kQkSlots = 2;                 // Q + K of an item (4 tiles), free once S = Q K^T is done
constexpr int kVSlots = 2;                  // V of an item (2 tiles), free once O = P V is done
constexpr uint32_t kQkSlot = 4 * kTile;
constexpr uint32_t kVSlot = 2 * kTile;
constexpr uint32_t kOffV = kQkSlots * kQkSlot;
constexpr uint32_t kStage = 4096;          // per softmax warp: 32 rows x 128 B of O (bf16), swizzled
constexpr uint32_t kOffStage = kOffV + kVSlots * kVSlot;
constexpr uint32_t kOffBar = kOffStage + 8 * kStage;
constexpr int kWG = 128;                    // a softmax / epilogue warpgroup
constexpr int kQkWarp = 8;                  // TMA loads of Q and K
constexpr int kVWarp = 9;                   // TMA loads of V
constexpr int kMmaWarp = 10;                // tcgen05.mma issue
constexpr int kThreads = 352;               // warpgroups 0 and 1 (warps 0-7) + 3 single warps
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024 /*alignment slack*/;

struct TesaTcParams {
    int T, H, W, nh;
    int Tw, Sw;
    int sw_log2;        // log2(Sw) when Sw is a power of two, else -1
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

// grid coordinates of box row r (r = (tt*Sw + hh)*Sw + ww)
__device__ __forceinline__ void row_coords(const TesaTcParams &p, const Item &it, int r, int &tt, int &hh, int &ww)
{
    if (p.sw_log2 >= 0) {
        const int l = p.sw_log2;
        tt = it.t0 + (r >> (2 * l));
        hh = it.h0 + ((r >> l) & (p.Sw - 1));
        ww = it.w0 + (r & (p.Sw - 1));
    } else {
        const int ss = p.Sw * p.Sw;
        tt = it.t0 + r / ss;
        hh = it.h0 + (r / p.Sw) % p.Sw;
        ww = it.w0 + r % p.Sw;
    }
}

// is box row r inside the grid?
__device__ __forceinline__ bool row_in_grid(const TesaTcParams &p, const Item &it, int r)
{
    int tt, hh, ww;
    row_coords(p, it, r, tt, hh, ww);
    return tt >= 0 && tt < p.T && hh >= 0 && hh < p.H && ww >= 0 && ww < p.W;
}

// Persistent CTA (one per SM) walking its share of the items.
//   QK warp   : TMA Q and K of item i into QK slot i % 2 once S of item i-2 is done
//   V warp    : TMA V of item i into V slot i % 2 once P V of item i-2 is done
//   MMA warp  : S(i) = Q K^T into the S columns of TMEM buffer i % 2 once P V of
//               item i-2 has consumed the P held there; then, one item behind,
//               O = P V with P taken from TMEM (P overwrites S), once the
//               epilogue of item i-2 has read the O columns
//   warpgroup g takes items i % 2 == g: softmax of S into P (bf16, in TMEM),
//               then the epilogue O / rowsum -> global
__global__ void __launch_bounds__(kThreads, 1)
    tesa_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, TesaTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *qk_full = bars;        // [2]
    uint64_t *qk_empty = bars + 2;   // [2] S done
    uint64_t *v_full = bars + 4;     // [3]
    uint64_t *v_empty = bars + 7;    // [3] P V done
    uint64_t *s_full = bars + 10;    // [2] S in TMEM buffer
    uint64_t *p_full = bars + 12;    // [2] P in TMEM buffer (128 arrivals)
    uint64_t *o_full = bars + 14;    // [2] O in TMEM buffer
    uint64_t *t_empty = bars + 16;   // [2] TMEM buffer read out (128 arrivals)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 18);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_items = p.items > (int)blockIdx.x ? (p.items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&qk_full[i], 1);
            tc::mbar_init(&qk_empty[i], 1);
            tc::mbar_init(&s_full[i], 1);
            tc::mbar_init(&p_full[i], kWG);
            tc::mbar_init(&o_full[i], 1);
            tc::mbar_init(&t_empty[i], kWG);
        }
        for (int i = 0; i < kVSlots; ++i) {
            tc::mbar_init(&v_full[i], 1);
            tc::mbar_init(&v_empty[i], 1);
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
    if (warp == kQkWarp) {
        for (int i = 0; i < n_items; ++i) {
            const int s = i & 1;
            if (i >= 2 && !wait_all(&qk_empty[s], ((i >> 1) - 1) & 1)) break;
            if (lane == 0) {
                const Item it = item_of(p, i);
                uint8_t *st = smem + s * kQkSlot;
                tc::mbar_expect_tx(&qk_full[s], kQkSlot);
                for (int half = 0; half < 2; ++half) {
                    tc::tma_load_5d(st + half * kTile, &mq, &qk_full[s], half * 64, it.head, it.w0, it.h0, it.t0);
                    tc::tma_load_5d(st + (2 + half) * kTile, &mk, &qk_full[s], half * 64, it.head, it.w0, it.h0, it.t0);
                }
            }
            __syncwarp();
        }
    } else if (warp == kVWarp) {
        for (int i = 0; i < n_items; ++i) {
            const int s = i % kVSlots;
            if (i >= kVSlots && !wait_all(&v_empty[s], ((i / kVSlots) - 1) & 1)) break;
            if (lane == 0) {
                const Item it = item_of(p, i);
                uint8_t *st = smem + kOffV + s * kVSlot;
                tc::mbar_expect_tx(&v_full[s], kVSlot);
                for (int half = 0; half < 2; ++half)
                    tc::tma_load_5d(st + half * kTile, &mv, &v_full[s], half * 64, it.head, it.w0, it.h0, it.t0);
            }
            __syncwarp();
        }
    } else if (warp == kMmaWarp) {
        const uint32_t id_s = tc::idesc_bf16(128, 128, 0, 0);
        const uint32_t id_o = tc::idesc_bf16(128, 128, 0, 1);
        auto issue_s = [&](int i) -> bool {
            const int b = i & 1;
            const uint32_t ph = (i >> 1) & 1;
            if (!wait_all(&qk_full[b], ph)) return false;
            // S overwrites P of item i-2: wait until P V of that item is done
            if (i >= 2 && !wait_all(&o_full[b], ph ^ 1)) return false;
            tc::tc_fence_after();
            if (lane == 0) {
                const uint32_t q0 = tc::smem_u32(smem + b * kQkSlot), k0 = q0 + 2 * kTile;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * kTile + (k & 3) * 32;
                    tc::mma_bf16(tmem + b * 256, tc::sdesc_sw128(q0 + off, 16, 1024), tc::sdesc_sw128(k0 + off, 16, 1024),
                                 id_s, k > 0);
                }
                tc::mma_commit(&s_full[b]);
                tc::mma_commit(&qk_empty[b]);
            }
            __syncwarp();
            return true;
        };
        if (n_items > 0 && issue_s(0)) {
            for (int i = 0; i < n_items; ++i) {
                if (i + 1 < n_items && !issue_s(i + 1)) break;
                const int b = i & 1, vs = i % kVSlots;
                if (!wait_all(&p_full[b], (i >> 1) & 1)) break;
                if (!wait_all(&v_full[vs], (i / kVSlots) & 1)) break;
                // O overwrites O of item i-2: wait until its epilogue has read it
                if (i >= 2 && !wait_all(&t_empty[b], ((i >> 1) & 1) ^ 1)) break;
                tc::tc_fence_after();
                if (lane == 0) {
                    const uint32_t v0 = tc::smem_u32(smem + kOffV + vs * kVSlot);
                    const uint32_t tP = tmem + b * 256;  // P (bf16 pairs) over S
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_bf16_tmem_a(tmem + b * 256 + 128, tP + k * 8, tc::sdesc_sw128(v0 + k * 2048, kTile, 1024),
                                            id_o, k > 0);
                    tc::mma_commit(&o_full[b]);
                    tc::mma_commit(&v_empty[vs]);
                }
                __syncwarp();
            }
        }
    } else if (warp < 8) {
        // ---- warpgroup g handles the items i with i % 2 == g (TMEM buffer g)
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
            const bool all_keys = (kmask[0] & kmask[1] & kmask[2] & kmask[3]) == 0xffffffffu;
            if (!wait_all(&s_full[g], ph)) break;
            tc::tc_fence_after();
            // the whole S row in registers (one TMEM round trip)
            float sv[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(tc::tmem_addr(tS, lane_base, c * 32), sv[c]);
            tc::tmem_wait_ld();
            if (!all_keys) {
                // keys outside the grid (zero-filled rows) take no weight
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (!((kmask[c] >> j) & 1u)) sv[c][j] = -INFINITY;
            }
            // row maximum over eight independent chains
            float m8[8];  // two more values per chain per three-input max
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = fmaxf(sv[0][u], sv[0][u + 8]);
#pragma unroll
            for (int i = 16; i < 128; i += 16)
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    m8[u] = tc::fmax3(m8[u], sv[i >> 5][(i & 31) + u], sv[i >> 5][(i & 31) + u + 8]);
            const float mx = fmaxf(tc::fmax3(m8[0], m8[1], m8[2]),
                                   tc::fmax3(tc::fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
            // P = 2^(S log2(e)/sqrt(d) - max') as bf16 pairs into TMEM columns
            // 16c .. 16c+15 (over S columns already read), and the row sum
            const float mxs = mx * p.scale_log2;
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-mxs, -mxs);
            float s8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) s8[u] = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {  // exponent arguments as packed fp32 pairs
                    const float2 t = tc::fma_f32x2(make_float2(sv[c][2 * j], sv[c][2 * j + 1]), sc2, nm2);
                    const float e0 = tc::ex2_approx(t.x), e1 = tc::ex2_approx(t.y);
                    s8[(2 * j) & 7] += e0;
                    s8[(2 * j + 1) & 7] += e1;
                    pk[j] = tc::pack_bf16(e0, e1);
                }
                tc::tmem_st16(tc::tmem_addr(tS, lane_base, c * 16), pk);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&p_full[g]);
            const float sum = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
            const float inv = 1.f / sum;

            // epilogue: O row / sum -> global, once P V is done. Each warp stages
            // its 32 rows, 64 head dims at a time, in shared memory and writes
            // them back as whole 128-byte lines (four rows per store instruction).
            if (!wait_all(&o_full[g], ph)) break;
            tc::tc_fence_after();
            int tt, hh, ww;
            row_coords(p, it, row, tt, hh, ww);
            const bool qvalid = tt >= 0 && tt < p.T && hh >= 0 && hh < p.H && ww >= 0 && ww < p.W;
            const size_t my_off = qvalid ? ((((size_t)tt * p.H + hh) * p.W + ww) * p.nh + it.head) * 128 : ~(size_t)0;
            uint8_t *stage = smem + kOffStage + warp * kStage;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float o[2][32];
                tc::tmem_ld32(tc::tmem_addr(tO, lane_base, hf * 64), o[0]);
                tc::tmem_ld32(tc::tmem_addr(tO, lane_base, hf * 64 + 32), o[1]);
                tc::tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int u = q >> 2, c0 = (q & 3) * 8;
                    uint4 v;
                    const float2 inv2 = make_float2(inv, inv);  // packed fp32 pairs
                    const float2 o0 = tc::mul_f32x2(make_float2(o[u][c0 + 0], o[u][c0 + 1]), inv2);
                    const float2 o1 = tc::mul_f32x2(make_float2(o[u][c0 + 2], o[u][c0 + 3]), inv2);
                    const float2 o2 = tc::mul_f32x2(make_float2(o[u][c0 + 4], o[u][c0 + 5]), inv2);
                    const float2 o3 = tc::mul_f32x2(make_float2(o[u][c0 + 6], o[u][c0 + 7]), inv2);
                    v.x = tc::pack_bf16(o0.x, o0.y);
                    v.y = tc::pack_bf16(o1.x, o1.y);
                    v.z = tc::pack_bf16(o2.x, o2.y);
                    v.w = tc::pack_bf16(o3.x, o3.y);
                    *reinterpret_cast<uint4 *>(stage + lane * 128 + ((q ^ (lane & 7)) << 4)) = v;
                }
                __syncwarp();
                // lane l writes 16-byte piece (l % 8) of rows 4k + l / 8
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int rr = k * 4 + (lane >> 3), q = lane & 7;
                    const size_t off = __shfl_sync(0xffffffffu, my_off, rr);
                    const uint4 v = *reinterpret_cast<const uint4 *>(stage + rr * 128 + ((q ^ (rr & 7)) << 4));
                    if (off != ~(size_t)0) *reinterpret_cast<uint4 *>(p.out + off + hf * 64 + q * 8) = v;
                }
                __syncwarp();
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
// (batch element of a (T, H, W, nh, 128) bf16 tensor) -> 5-D map, box = 64 x 1 x Sw x Sw x Tw
bool make_map(CUtensorMap *m, const void *base, const TesaArgs &a)
{
    const uint64_t e = 2;
    const uint64_t dims[5] = {128, (uint64_t)a.nh, (uint64_t)a.W, (uint64_t)a.H, (uint64_t)a.T};
    const uint64_t strides[4] = {128 * e, (uint64_t)a.nh * 128 * e, (uint64_t)a.W * a.nh * 128 * e,
                                 (uint64_t)a.H * a.W * a.nh * 128 * e};
    const uint32_t box[5] = {64, 1, (uint32_t)a.Sw, (uint32_t)a.Sw, (uint32_t)a.Tw};
    return tmap_bf16_5d(m, base, dims, strides, box);
}

}  // namespace

bool tesa_tc_supported(const TesaArgs &a)
{
    return a.bf16 && a.d == 128 && a.Tw * a.Sw * a.Sw == 128 && a.Sw <= 128 && a.Tw <= 128 &&
           (size_t)a.nwt * a.nwh * a.nww * a.nh < ((size_t)1 << 31) &&
           tmap_available();
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
    p.sw_log2 = -1;
    for (int l = 0; l < 8; ++l)
        if ((1 << l) == a.Sw) p.sw_log2 = l;
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
