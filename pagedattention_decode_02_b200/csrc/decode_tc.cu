// Tensor-core decode of grouped query heads (placeholder until the kernel lands).
#include "decode_launch.h"
#include "pool.h"

namespace pkv {

void pool_init_device_extras(pkv_pool* p) { p->has_tmaps = false; }

bool tensor_path_supported(int, int, int, int, int) { return false; }

cudaError_t launch_decode_tensor(const DecodeParams&, const void*, const void*, int, int,
                                 cudaStream_t, cudaEvent_t) {
    return cudaErrorNotSupported;
}

}  // namespace pkv
