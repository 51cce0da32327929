// decode_i8.cu -- the decode kernels of the INT8 output: instantiations of decode_device.cuh,
// compiled on their own so the library builds in parallel.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchI8 = make_launchers<kOutI8>();
}  // namespace dec
}  // namespace ep
