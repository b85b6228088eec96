// hgrn2_all.cu -- single translation unit of libhgrn2.so.
//
// The kernels share the device-side status word and counters defined in
// api.cu; compiling them as one unit keeps those references plain (no
// relocatable device code or device link step).
#include "api.cu"
#include "simt.cu"
#include "step.cu"
#include "varlen.cu"
#include "scalar.cu"
#include "selftest.cu"
#include "wide.cu"
#include "seqpar.cu"
#include "tc_fwd.cu"
#include "tc_bwd.cu"
