// Types shared by the kernels of this library.
#pragma once
#include <cstdint>

namespace intattn {

// Integer parameters of one head, derived on the host (see intattn.h):
// index multiplier M and shift s, gap clip D, requantisation Mo / so, which
// of the call's LUTs (one per distinct clip threshold) the head uses, and the
// zero-point of its V codes (0: int8 V).
struct HeadParamsDev {
  int32_t M, s, D, Mo, so, lut, zv;
};

// The V zero-point enters the output as acc = sum_j P_j v_j - zv sum_j P_j.
// The tensor core subtracts zv sum_j P_j through one more K = 32 MMA per
// partial owner group: a "correction" P tile whose u8 entries (a0 .. a4)
// satisfy a0 + 128 (a1 + a2 + a3 + a4) = zv * (the owner's share of
// sum_j P_j), against a constant s8 tile whose rows hold -1 (row 0 of an
// owner's group) and -128 (rows 1 .. 4).  sum_j P_j <= 510 over a row, so
// zv * share < 2^17 and the split below always fits.
__device__ __forceinline__ void zv_correction_bytes(int32_t n, uint32_t& w0, uint32_t& w1) {
  const uint32_t a0 = static_cast<uint32_t>(n) & 127u;
  uint32_t rest = static_cast<uint32_t>(n) >> 7;  // <= 1016: four bytes of at most 255
  uint32_t a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[i] = rest < 255u ? rest : 255u;
    rest -= a[i];
  }
  w0 = a0 | (a[0] << 8) | (a[1] << 16) | (a[2] << 24);
  w1 = a[3];
}

}  // namespace intattn
