// decode_e4m3row.cu -- the decode kernels of the FP8 container with a per-row scale (E4M3 payload
// plus one fp32 scale per row): instantiations of decode_device.cuh, compiled on their own for a
// parallel build.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchE4M3Row = make_launchers<kOutE4M3Row>();
}  // namespace dec
}  // namespace ep
