// Quantisation prologue: FP16 / BF16 activations -> int8 codes with a
// dynamic symmetric scale per tensor or per head.
//
// IntAttention's integer pipeline starts from int8 Q, K, V; the forum page
// "IntAttention：面向边缘设备的纯整数注意力推理加速方案", section 动态量化策略,
// describes choosing the quantisation range of each layer (or head) from the
// live activations.  Definition computed here (identical to the numpy
// oracle): amax = max |x| over the tensor or over one head [B, L, d] slice;
// s = amax / 127 and inv = min(127 / amax, FLT_MAX) (IEEE fp32 divisions),
// s = inv = 1 if amax = 0; code = clamp(rint(x * inv), -127, 127) with the
// fp32 product rounded to nearest and rint rounding half to even.
// Zero-point 0.
//
// Three launches per tensor: quant_amax (per-CTA max |x| of a slice chunk,
// atomicMax on the float bits, which order like the unsigned integers for
// values >= 0), quant_codes (each CTA derives s from amax and writes the
// codes), quant_scales (amax -> s in place).  The caller's scale buffer
// holds amax between the launches; it is zeroed by a memset first.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace intattn {

struct QuantArgs {
  const void* x;     // [B, H, L, d] fp16 or bf16
  int8_t* out;       // [B, H, L, d]
  uint32_t* amax;    // [H] or [1]: the caller's float scale buffer, used as bits
  int64_t slice;     // L * d elements of one (b, h)
  int32_t H, per_head, bf16, chunks;  // chunks: CTAs per (b, h) slice
};

namespace quant {

constexpr int kThreads = 256;
constexpr int kVec = 8;                          // elements per 16-byte load
constexpr int kIters = 16;                       // loads per thread and CTA
constexpr int kChunkElems = kThreads * kVec * kIters;  // 32768 elements per CTA

__device__ __forceinline__ void to_float8(uint4 v, bool bf16, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (bf16) {
      f[2 * i] = __uint_as_float(w[i] << 16);            // bf16 = high half of an fp32
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      f[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
      f[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
    }
  }
}

__device__ __forceinline__ float scale_of(uint32_t amax_bits) {
  const float s = __fdiv_rn(__uint_as_float(amax_bits), 127.0f);
  return s == 0.0f ? 1.0f : s;
}
// 127 / amax, capped at the largest float (an amax below 127 / FLT_MAX would
// overflow it)
__device__ __forceinline__ float inv_scale_of(uint32_t amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  return amax == 0.0f ? 1.0f : fminf(__fdiv_rn(127.0f, amax), 3.402823466e38f);
}

// grid (chunks, B*H)
__global__ void __launch_bounds__(kThreads) quant_amax_kernel(const __grid_constant__ QuantArgs a) {
  const int bh = blockIdx.y;
  const int64_t e0 = static_cast<int64_t>(blockIdx.x) * kChunkElems;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + bh * a.slice);
  float m = 0.0f;
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int64_t e = e0 + (static_cast<int64_t>(it) * kThreads + threadIdx.x) * kVec;
    if (e < a.slice) {
      float f[8];
      to_float8(__ldg(src + e / kVec), a.bf16, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
    const int slot = a.per_head ? bh % a.H : 0;
    atomicMax(a.amax + slot, __float_as_uint(m));
  }
}

// grid (chunks, B*H)
__global__ void __launch_bounds__(kThreads) quant_codes_kernel(const __grid_constant__ QuantArgs a) {
  const int bh = blockIdx.y;
  const int64_t e0 = static_cast<int64_t>(blockIdx.x) * kChunkElems;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + bh * a.slice);
  uint2* dst = reinterpret_cast<uint2*>(a.out + bh * a.slice);
  const float inv = inv_scale_of(__ldcg(a.amax + (a.per_head ? bh % a.H : 0)));
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int64_t e = e0 + (static_cast<int64_t>(it) * kThreads + threadIdx.x) * kVec;
    if (e < a.slice) {
      float f[8];
      to_float8(__ldg(src + e / kVec), a.bf16, f);
      uint32_t b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int q = __float2int_rn(__fmul_rn(f[i], inv));
        q = q > 127 ? 127 : (q < -127 ? -127 : q);
        b[i] = static_cast<uint32_t>(q) & 0xFFu;
      }
      dst[e / kVec] = make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                                 b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
    }
  }
}

// one CTA: amax bits -> the float scale, in place
__global__ void quant_scales_kernel(uint32_t* amax, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) amax[i] = __float_as_uint(scale_of(amax[i]));
}

}  // namespace quant
}  // namespace intattn
