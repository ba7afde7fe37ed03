// nvfp4_runtime.h -- host/device definitions shared by the library's translation units
// (not part of the C ABI).
#pragma once

#include <cstdint>

namespace nvfp4 {

// The caller's NVFP4_WORKSPACE_BYTES of device memory.  It starts zeroed; every kernel
// that uses it leaves acc / arrived / departed zeroed again, and `error` keeps
// NVFP4_ERR_TIMEOUT once a bounded device-side wait gave up (nvfp4_workspace_check
// reads and clears it).
struct Workspace {
    unsigned acc;       // running max |x| as fp32 bits
    unsigned arrived;   // CTAs that have finished their share of the amax
    unsigned departed;  // CTAs that have left the grid barrier (fused kernel)
    unsigned error;     // NVFP4_ERR_TIMEOUT once a bounded wait gave up
    unsigned pad[60];
};
static_assert(sizeof(Workspace) == 256, "NVFP4_WORKSPACE_BYTES");

// Counts one kernel launch of this library (nvfp4_kernel_launch_count).
void note_launch();

}  // namespace nvfp4
