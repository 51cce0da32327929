// decode_bf16.cu -- the decode kernels of the BF16 output: instantiations of decode_device.cuh,
// compiled on their own so the library builds in parallel.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchBF16 = make_launchers<kOutBF16>();
}  // namespace dec
}  // namespace ep
