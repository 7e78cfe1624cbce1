// Host-side construction of TMA tensor maps (bf16, 128-byte swizzle, zero fill
// out of bounds). The driver's encoder is reached through the runtime's
// driver entry point, so the library does not link the driver library.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace mate {

// True if the driver's tensor-map encoder is available.
bool tmap_available();

// 5-D bf16 map: dims[0] elements contiguous, strides in bytes for dims 1..4,
// box[0..4] elements per dimension. False if the encoder rejects the map.
bool tmap_bf16_5d(CUtensorMap *m, const void *base, const uint64_t dims[5], const uint64_t strides[4],
                  const uint32_t box[5]);

// Rows of one 128-position sub-chunk of a Rotary-Major-Scan order as a TMA box.
// The scan's axes, fastest first, become map dimensions 2, 3, 4; the sub-chunk
// starting at scan position s sits at (s % n0, (s / n0) % n1, s / (n0 n1)).
struct ScanBox {
    int ok;               // 0: the sub-chunks of this grid and order are not boxes
    int n[3];             // axis lengths, fastest first
    int64_t stride[3];    // axis strides in tokens
    uint32_t box[3];      // box extent per axis (product 128)
};
ScanBox scan_box(int mode, int T, int H, int W);

}  // namespace mate
