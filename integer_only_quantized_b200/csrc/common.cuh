// Types shared by the kernels of this library.
#pragma once
#include <cstdint>

namespace intattn {

// Integer parameters of one head, derived on the host (see intattn.h):
// index multiplier M and shift s, gap clip D, requantisation Mo / so, and
// which of the call's LUTs (one per distinct clip threshold) the head uses.
struct HeadParamsDev {
  int32_t M, s, D, Mo, so, lut;
};

}  // namespace intattn
