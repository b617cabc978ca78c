// Host-side launcher of the cache-append kernels (internal; the public call is
// mla_cache_append in include/mla.h). Arguments are validated by the caller.
#pragma once

#include <cuda_runtime.h>

#include "../../include/mla.h"

namespace mla {

cudaError_t launch_cache_append(const mla_append_args* a, cudaStream_t st);

}  // namespace mla
