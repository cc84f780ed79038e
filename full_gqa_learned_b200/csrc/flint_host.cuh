// Host-side helpers shared by the library's translation units: the error
// text of the calling thread, the driver's tensor-map encoder and the
// once-per-device setup (architecture check, SM count).
#pragma once
#include <cuda.h>

#include "../../include/flint_attn.h"

namespace flint {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Records printf-style text as the calling thread's last error; returns s.
flint_status_t fail(flint_status_t s, const char* fmt, ...);
// cuTensorMapEncodeTiled through the runtime's driver entry point.
flint_status_t get_encoder(EncodeTiledFn* fn);
// Checks for an sm_100 device, sets the attention kernel's shared-memory
// limit once per device and returns its SM count.
flint_status_t device_setup(int* sms);

}  // namespace flint
