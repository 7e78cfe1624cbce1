// TMA tensor maps: see tmap.h.
#include "tmap.h"

#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mate.h"

namespace mate {

namespace {

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

}  // namespace

bool tmap_available() { return encode_fn() != nullptr; }

bool tmap_bf16_5d(CUtensorMap *m, const void *base, const uint64_t dims[5], const uint64_t strides[4],
                  const uint32_t box[5])
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < 5; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
    }
    for (int i = 0; i < 4; ++i) st[i] = strides[i];
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), d, st, bx, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

ScanBox scan_box(int mode, int T, int H, int W)
{
    // axes fastest first, as the scan orders of rms_grid_offset walk them
    ScanBox sb = {};
    const int64_t sw = 1, sh = W, st = (int64_t)H * W;
    int n[3];
    int64_t s[3];
    switch (mode) {
    case MATE_SCAN_SR:  // (t, h, w): w fastest
        n[0] = W; s[0] = sw; n[1] = H; s[1] = sh; n[2] = T; s[2] = st;
        break;
    case MATE_SCAN_SC:  // (t, w, h): h fastest
        n[0] = H; s[0] = sh; n[1] = W; s[1] = sw; n[2] = T; s[2] = st;
        break;
    case MATE_SCAN_TR:  // (h, w, t): t fastest
        n[0] = T; s[0] = st; n[1] = W; s[1] = sw; n[2] = H; s[2] = sh;
        break;
    case MATE_SCAN_ZZ:  // rows alternate direction: no sub-chunk is a box of the grid
        return sb;
    default:            // MATE_SCAN_TC (w, h, t): t fastest
        n[0] = T; s[0] = st; n[1] = H; s[1] = sh; n[2] = W; s[2] = sw;
        break;
    }
    uint32_t b[3] = {1, 1, 1};
    if (n[0] % 128 == 0) {
        b[0] = 128;
    } else if (128 % n[0] == 0 && n[1] % (128 / n[0]) == 0) {
        b[0] = n[0];
        b[1] = 128 / n[0];
    } else if (128 % (n[0] * n[1]) == 0 && n[2] % (128 / (n[0] * n[1])) == 0) {
        b[0] = n[0];
        b[1] = n[1];
        b[2] = 128 / (n[0] * n[1]);
    } else {
        return sb;
    }
    sb.ok = 1;
    for (int i = 0; i < 3; ++i) {
        sb.n[i] = n[i];
        sb.stride[i] = s[i];
        sb.box[i] = b[i];
    }
    return sb;
}

}  // namespace mate
