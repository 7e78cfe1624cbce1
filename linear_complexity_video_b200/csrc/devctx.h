// Identity of the current CUDA context, for caches of device addresses that
// belong to one context (the device image of this library is loaded once per
// context: destroying a device's primary context with cudaDeviceReset unloads
// it, and the next context may place its variables elsewhere).
#pragma once

namespace mate {

// Unique id of the calling thread's current context (cuCtxGetId, reached
// through the runtime's driver entry points). Returns 0 if it cannot be read;
// callers then fall back to keying their cache by device only.
unsigned long long current_context_id();

}  // namespace mate
