// placeholder
#include "kvq_internal.h"
namespace kvq {
size_t attend_workspace_bytes(int, int, int, int, int) { return 256; }
kvq_status launch_attend_int4(const kvq_plan*, const kvq_plan*, const uint16_t*, const uint8_t*, const uint16_t*,
                              const uint8_t*, const uint16_t*, int, int, int, int, const int32_t*, int, float,
                              uint16_t*, void*, size_t, cudaStream_t) { return KVQ_ERR_UNSUPPORTED; }
kvq_status launch_attend_fp16(const uint16_t*, const uint16_t*, const uint16_t*, int, int, int, int, int,
                              const int32_t*, int, float, uint16_t*, void*, size_t, cudaStream_t) { return KVQ_ERR_UNSUPPORTED; }
uint32_t attend_error_flags(bool) { return 0; }
}
