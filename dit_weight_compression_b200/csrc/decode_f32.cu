// decode_f32.cu -- the decode kernels of the FP32 output: instantiations of decode_device.cuh,
// compiled on their own so the library builds in parallel.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchF32 = make_launchers<kOutF32>();
}  // namespace dec
}  // namespace ep
