// tma_host.h -- host side of the TMA tensor maps: the driver's
// cuTensorMapEncodeTiled, looked up once through the runtime (no link
// dependency on libcuda beyond what the runtime loads).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

namespace qlora {

// nullptr when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace qlora
