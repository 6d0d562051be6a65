// Entry points whose kernels are not wired yet return METIS_ERR_UNSUPPORTED.
#include "abi_common.h"

extern "C" {

metis_status metis_split(const void*, int32_t, int64_t, int64_t, int64_t, const metis_split_params*,
                         float*, float*, float*, metis_fp4_tensor*, metis_fp4_tensor*,
                         metis_fp4_tensor*, metis_fp4_tensor*, float*, int32_t*, void*, size_t*,
                         int32_t*, void*) {
  return METIS_ERR_UNSUPPORTED;
}

metis_status averis_split(const void*, int32_t, int64_t, int64_t, int64_t, int32_t, float*,
                          metis_fp4_tensor*, metis_fp4_tensor*, metis_fp4_tensor*, float*, void*,
                          size_t*, int32_t*, void*) {
  return METIS_ERR_UNSUPPORTED;
}

}  // extern "C"
