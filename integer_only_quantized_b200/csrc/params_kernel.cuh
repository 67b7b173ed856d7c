// Integer parameters of every head derived on the device, from quantisation
// scales that a preceding kernel left in device memory, so that quantising
// fp16 / bf16 activations and running the integer forward need no round
// trip to the host.
//
// The steps are those of the host derivation in intattn.cu (and of the
// definition in intattn.h), in IEEE double in the same order: correctly
// rounded multiply, divide and square root, and exact ldexp, frexp and
// llround, so the results are the host's bit for bit.
#pragma once
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace intattn {

// set in the device error word when a derived parameter is out of range
constexpr unsigned int kErrParamRange = 2u;

struct DeriveArgs {
  const float* s_q;      // device: quantisation scales, H entries (per head) or 1
  const float* s_k;
  const float* s_v;
  const int32_t* z_v;    // device: V zero-points (asymmetric V codes), or null
  HeadParamsDev* hp;     // device out: per head (or entry 0)
  uint32_t* status;      // device out: 0, or kErrParamRange
  int32_t n;             // entries: H (per head) or 1
  int32_t d;
  float s_o[INTATTN_MAX_HEADS];   // output scale per entry (host values)
  float clip[INTATTN_MAX_HEADS];  // clip threshold per entry
  int32_t lut[INTATTN_MAX_HEADS]; // exp table index per entry
};

namespace params {

__device__ __forceinline__ bool index_params(double s_q, double s_k, int d, double c, HeadParamsDev& hp) {
  if (!isfinite(s_q) || !isfinite(s_k) || !(s_q > 0.0) || !(s_k > 0.0)) return false;
  const double alpha = (s_q * s_k) / sqrt(static_cast<double>(d));
  const double steps = (alpha * 31.0) / c;
  int shift = 26;
  long long mult = llround(ldexp(steps, shift));
  while (shift > 1 && mult > (1ll << 24)) {
    --shift;
    mult = llround(ldexp(steps, shift));
  }
  if (mult < 1 || mult > (1ll << 24) || mult > (1ll << shift)) return false;
  const long long half_steps = 61ll << (shift - 1);
  hp.M = static_cast<int32_t>(mult);
  hp.s = shift;
  hp.D = static_cast<int32_t>((half_steps + mult - 1) / mult);
  return true;
}

__device__ __forceinline__ bool requant_params(double s_v, double s_o, HeadParamsDev& hp) {
  if (!isfinite(s_v) || !(s_v > 0.0)) return false;
  int e = 0;
  const double f = frexp(s_v / (255.0 * s_o), &e);
  long long mo = llround(f * 2147483648.0);
  if (mo == (1ll << 31)) {
    mo = 1ll << 30;
    ++e;
  }
  const int so = 31 - e;
  if (so < 1 || so > 62) return false;
  hp.Mo = static_cast<int32_t>(mo);
  hp.so = so;
  return true;
}

// one CTA: thread i derives entry i
__global__ void derive_params_kernel(const __grid_constant__ DeriveArgs a) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < a.n; i += blockDim.x) {
    HeadParamsDev hp{};
    const bool ok = index_params(a.s_q[i], a.s_k[i], a.d, a.clip[i], hp) && requant_params(a.s_v[i], a.s_o[i], hp);
    hp.lut = a.lut[i];
    hp.zv = a.z_v ? a.z_v[i] : 0;
    a.hp[i] = hp;
    if (!ok) atomicOr(&bad, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *a.status = bad ? kErrParamRange : 0u;
    if (bad) atomicOr(&g_device_error, kErrParamRange);
  }
}

}  // namespace params
}  // namespace intattn
