// Chunked prefill over the paged cache (tcgen05).  Entry point only for now.
#include "pa_internal.h"

extern "C" pa_status pa_prefill_paged(void*, const void*, const void*, const void*,
                                      const int32_t*, const int32_t*, const int32_t*, float,
                                      int, int, int, int, int, int, int, int, pa_dtype,
                                      pa_dtype, float, float, int32_t*, void*) {
  return PA_ERR_UNSUPPORTED;
}
