// Chunked prefill over the paged cache (tensor-core kernel follows).
#include "pa_device.cuh"
#include "pa_host.h"

extern "C" size_t pa_chunked_prefill_workspace_size(int, int, int, int, int) { return 0; }

extern "C" pa_status pa_chunked_prefill(void*, const void*, const void*, const void*,
                                        const int32_t*, int, const int32_t*, const int32_t*, int,
                                        int, int, int, int, float, int, int, int, void*, size_t,
                                        pa_dtype, void*) {
  pa::set_launch_count(0);
  return PA_ERR_UNSUPPORTED;
}
