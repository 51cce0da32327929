// decode_fp16.cu -- the decode kernels of the FP16 output: instantiations of decode_device.cuh,
// compiled on their own so the library builds in parallel.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchFP16 = make_launchers<kOutFP16>();
}  // namespace dec
}  // namespace ep
