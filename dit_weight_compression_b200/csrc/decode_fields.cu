// decode_fields.cu -- the decode kernel of the fields test hook (the coset bit and eight fields of
// every vector): instantiations of decode_device.cuh, compiled on their own for a parallel build.
#include "decode_device.cuh"

namespace ep {
namespace dec {
const Launchers kLaunchFields = make_launchers<kOutFields>();
}  // namespace dec
}  // namespace ep
