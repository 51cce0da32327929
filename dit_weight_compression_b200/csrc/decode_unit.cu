// decode_unit.cu -- the decode kernels of one output container with one table layout:
// instantiations of decode_device.cuh.  The build compiles this file once per (container, layout)
// pair, with -DEP_UNIT_OUT=<container number, as in OutKind> and -DEP_UNIT_LAY=<10, 12, 13 or 14>,
// so the kernels compile in parallel; each object defines the launch table kLaunch_<out>_<lay>.
#include "decode_device.cuh"

#if !defined(EP_UNIT_OUT) || !defined(EP_UNIT_LAY)
#error "decode_unit.cu is compiled with -DEP_UNIT_OUT=<container> -DEP_UNIT_LAY=<layout>"
#endif

#define EP_UNIT_NAME2(o, l) kLaunch_##o##_##l
#define EP_UNIT_NAME(o, l) EP_UNIT_NAME2(o, l)

namespace ep {
namespace dec {
const Launchers EP_UNIT_NAME(EP_UNIT_OUT, EP_UNIT_LAY) = make_launchers<EP_UNIT_OUT, EP_UNIT_LAY>();
}  // namespace dec
}  // namespace ep
