// MATE composition on the 5th-generation tensor cores: the block output as the
// sum of the two branches projected to the model width,
//     out = y_MA W_MA^T + y_TE W_TE^T
// (paper review "LinGen ...", section 三, MATE: the MA-branch and the TE-branch
// together replace self-attention; the pages give no combination rule, and the
// two branch outputs have different widths (80 x 64 and 20 x 128 channels), so
// each is projected to the model width (2560, section 5.1) and the two are
// added). As one GEMM over the concatenated reduction dimension: the A operand
// walks y_MA's K_MA columns and then y_TE's K_TE columns, the B operand the
// matching rows of [W_MA | W_TE].
//
// Persistent, one CTA per SM, 192 threads:
//   warp 0    TMA loads of 128 x 64 A tiles and 256 x 64 B tiles into a 4-stage
//             ring (48 KB per stage, 128-byte swizzle, K-major);
//   warp 1    TMEM allocation and tcgen05.mma issue: per output tile of 128 x 256,
//             four M = 128, N = 256, K = 16 MMAs per stage into one of two TMEM
//             accumulators (2 x 256 columns), so that a tile's epilogue runs while
//             the next tile accumulates;
//   warps 2-5 the epilogue: TMEM -> registers -> bf16 -> a 128 x 64 staging tile
//             in the 128-byte swizzle (two, alternating) -> TMA store.
// Tiles go N fastest, so the CTAs at work share the A rows of a few M blocks in
// L2, and all of W stays in L2.
//
// Every wait is bounded (2 s); a wait that gives up records MATE_ERR_TIMEOUT and
// raises a CTA abort flag that makes every role leave its loop; the CTA then
// waits (bounded) for its copies and MMAs in flight and frees its TMEM.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

#include <algorithm>

namespace mate {

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr uint32_t kATile = kBM * kBK * 2;           // 16 KB
constexpr uint32_t kBTile = kBN * kBK * 2;           // 32 KB
constexpr uint32_t kStage = kATile + kBTile;         // 48 KB
constexpr uint32_t kOutTile = kBM * 64 * 2;          // 16 KB: 128 rows x 64 columns
constexpr uint32_t kOffStages = 0;
constexpr uint32_t kOffOut = kStages * kStage;       // 2 staging tiles
constexpr uint32_t kOffBar = kOffOut + 2 * kOutTile;
// full[4], empty[4], acc_full[2], acc_empty[2], drain; then the TMEM slot and the abort flag
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarAccFull = 2 * kStages, kBarAccEmpty = 2 * kStages + 2,
              kBarDrain = 2 * kStages + 4, kNumBars = 2 * kStages + 5;
constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "compose: shared memory");
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

struct ComposeGeo {
    int M, N, nk1, nk2;  // rows, columns, 64-wide K steps of the two parts
    int tiles_n, tiles;  // output tiles along N, in total
};

__global__ void __launch_bounds__(kThreads, 1)
    compose_tc_kernel(const __grid_constant__ CUtensorMap ma1, const __grid_constant__ CUtensorMap mb1,
                      const __grid_constant__ CUtensorMap ma2, const __grid_constant__ CUtensorMap mb2,
                      const __grid_constant__ CUtensorMap mo, ComposeGeo geo, int *err)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = geo.nk1 + geo.nk2;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            tc::mbar_init(&bars[kBarFull + i], 1);
            tc::mbar_init(&bars[kBarEmpty + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars[kBarAccFull + i], 1);
            tc::mbar_init(&bars[kBarAccEmpty + i], 128);
        }
        tc::mbar_init(&bars[kBarDrain], 1);
        tc::fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t it = 0;  // stage fills issued
            for (int t = blockIdx.x; t < geo.tiles && !*abort_flag; t += gridDim.x) {
                const int m0 = (t / geo.tiles_n) * kBM, n0 = (t % geo.tiles_n) * kBN;
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const int s = it % kStages;
                    const uint32_t round = it / kStages;
                    if (round > 0 && !tc::mbar_wait_or_abort(&bars[kBarEmpty + s], (round - 1) & 1u, err, abort_flag))
                        break;
                    uint8_t *sa = base + kOffStages + s * kStage, *sb = sa + kATile;
                    tc::mbar_expect_tx(&bars[kBarFull + s], kStage);
                    if (ks < geo.nk1) {
                        tc::tma_load_5d(sa, &ma1, &bars[kBarFull + s], ks * kBK, m0, 0, 0, 0);
                        tc::tma_load_5d(sb, &mb1, &bars[kBarFull + s], ks * kBK, n0, 0, 0, 0);
                    } else {
                        tc::tma_load_5d(sa, &ma2, &bars[kBarFull + s], (ks - geo.nk1) * kBK, m0, 0, 0, 0);
                        tc::tma_load_5d(sb, &mb2, &bars[kBarFull + s], (ks - geo.nk1) * kBK, n0, 0, 0, 0);
                    }
                }
            }
            // every load issued has landed before the CTA may leave (bounded)
            if (it > 0) {
                const uint32_t last = it - 1;
                tc::mbar_wait(&bars[kBarFull + last % kStages], (last / kStages) & 1u, nullptr);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issue ----------------
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16(kBM, kBN, 0, 0);
            uint32_t it = 0, tl = 0, committed = 0;
            for (int t = blockIdx.x; t < geo.tiles && !*abort_flag; t += gridDim.x, ++tl) {
                const uint32_t acc = tl & 1, use = tl >> 1;
                if (use > 0 && !tc::mbar_wait_or_abort(&bars[kBarAccEmpty + acc], (use - 1) & 1u, err, abort_flag))
                    break;
                tc::tc_fence_after();
                const uint32_t d = tmem + acc * kBN;
                bool ok = true;
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const int s = it % kStages;
                    if (!tc::mbar_wait_or_abort(&bars[kBarFull + s], (it / kStages) & 1u, err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t a0 = tc::smem_u32(base + kOffStages + s * kStage), b0 = a0 + kATile;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc::mma_bf16(d, tc::sdesc_sw128(a0 + kk * 32, 16, 1024), tc::sdesc_sw128(b0 + kk * 32, 16, 1024),
                                     idesc, ks > 0 || kk > 0);
                    tc::mma_commit(&bars[kBarEmpty + s]);  // the stage is free once these MMAs are done
                    ++committed;
                }
                if (!ok) break;
                tc::mma_commit(&bars[kBarAccFull + acc]);
            }
            // every MMA issued has completed before TMEM may be freed (bounded)
            if (committed > 0) {
                tc::mma_commit(&bars[kBarDrain]);
                tc::mbar_wait(&bars[kBarDrain], 0, nullptr);
            }
        }
    } else {
        // ---------------- epilogue: warps 2-5, TMEM lanes 32 (warp % 4) .. ----------------
        const int et = tid - 64;                        // 0..127
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const int row = (int)lane_base + lane;          // output row of the tile
        uint32_t tl = 0, chunks = 0;                    // tiles and 64-column chunks stored
        for (int t = blockIdx.x; t < geo.tiles; t += gridDim.x, ++tl) {
            const uint32_t acc = tl & 1, use = tl >> 1;
            if (!tc::mbar_wait_sleep(&bars[kBarAccFull + acc], use & 1u, err, abort_flag)) break;
            tc::tc_fence_after();
            const int m0 = (t / geo.tiles_n) * kBM, n0 = (t % geo.tiles_n) * kBN;
            for (int c = 0; c < kBN / 64 && n0 + 64 * c < geo.N; ++c, ++chunks) {
                uint32_t v[2][32];
                tc::tmem_ld32u(tc::tmem_addr(tmem + acc * kBN, lane_base, 64 * c), v[0]);
                tc::tmem_ld32u(tc::tmem_addr(tmem + acc * kBN, lane_base, 64 * c + 32), v[1]);
                tc::tmem_wait_ld();
                // the store that read this staging tile two chunks ago is done with it
                if (et == 0) tc::bulk_wait_read<1>();
                tc::named_sync(1, 128);
                uint8_t *stg = base + kOffOut + (chunks & 1) * kOutTile;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t *w = v[q >> 2] + 8 * (q & 3);
                    *reinterpret_cast<uint4 *>(stg + tc::sw128(row, q)) =
                        make_uint4(tc::pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                                   tc::pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                                   tc::pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                                   tc::pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7])));
                }
                tc::fence_proxy_async_smem();
                tc::named_sync(1, 128);
                if (et == 0) {
                    // rows past M fall outside the tensor and are not written
                    tc::tma_store_5d(&mo, stg, n0 + 64 * c, m0, 0, 0, 0);
                    tc::bulk_commit();
                }
            }
            // this accumulator may be overwritten by the tile after next
            tc::tc_fence_before();
            tc::mbar_arrive(&bars[kBarAccEmpty + acc]);
        }
        if (et == 0) tc::bulk_wait_all();
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

// Any N that keeps rows 16-byte aligned: the B tiles past N load as zeros and the
// output columns past N are clipped by the TMA store (a 64-column chunk that
// starts past N is skipped).
bool compose_tc_supported(const ComposeArgs &a)
{
    return a.M > 0 && a.N > 0 && a.N % 8 == 0 && a.K1 % kBK == 0 && a.K2 % kBK == 0 && a.K1 + a.K2 > 0;
}

cudaError_t launch_compose_tc(const ComposeArgs &a, cudaStream_t s)
{
    cudaError_t e = cudaFuncSetAttribute(compose_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if (!tmap_available()) return cudaErrorNotSupported;
    // 2-D row-major bf16 tensors as 5-D maps with unit trailing dimensions
    auto map2d = [](CUtensorMap *m, const void *p, uint64_t cols, uint64_t rows, uint32_t bc, uint32_t br) {
        const uint64_t dims[5] = {cols, rows, 1, 1, 1};
        const uint64_t strides[4] = {cols * 2, cols * rows * 2, cols * rows * 2, cols * rows * 2};
        const uint32_t box[5] = {bc, br, 1, 1, 1};
        return tmap_bf16_5d(m, p, dims, strides, box);
    };
    CUtensorMap ma1 = {}, mb1 = {}, ma2 = {}, mb2 = {}, mo = {};
    // a part with no columns still needs a valid map: it is never read
    const void *a2 = a.K2 ? a.y2 : a.y1, *b2 = a.K2 ? a.w2 : a.w1;
    const uint64_t k2 = a.K2 ? a.K2 : a.K1;
    const void *a1 = a.K1 ? a.y1 : a.y2, *b1 = a.K1 ? a.w1 : a.w2;
    const uint64_t k1 = a.K1 ? a.K1 : a.K2;
    if (!map2d(&ma1, a1, k1, a.M, kBK, kBM) || !map2d(&mb1, b1, k1, a.N, kBK, kBN) || !map2d(&ma2, a2, k2, a.M, kBK, kBM) ||
        !map2d(&mb2, b2, k2, a.N, kBK, kBN) || !map2d(&mo, a.out, a.N, a.M, 64, kBM))
        return cudaErrorInvalidValue;
    ComposeGeo geo;
    geo.M = a.M;
    geo.N = a.N;
    geo.nk1 = a.K1 / kBK;
    geo.nk2 = a.K2 / kBK;
    geo.tiles_n = (a.N + kBN - 1) / kBN;
    geo.tiles = ((a.M + kBM - 1) / kBM) * geo.tiles_n;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(geo.tiles, std::max(nsm, 1));
    Phase ph(a.phase ? a.phase : MATE_PHASE_COMPOSE, s);
    compose_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(ma1, mb1, ma2, mb2, mo, geo, a.err);
    return cudaGetLastError();
}

}  // namespace mate
