// decode_e4m3.cu -- the decode kernels of the FP8 E4M3 output: instantiations of decode_device.cuh,
// compiled on their own so the library builds in parallel.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchE4M3 = make_launchers<kOutE4M3>();
}  // namespace dec
}  // namespace ep
