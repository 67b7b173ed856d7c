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
// Two launches per tensor.  quant_zero clears the caller's scale buffer
// (which holds amax as float bits until the end) and the first 8 bytes of
// the code buffer (two grid-barrier counters until the end).  quant_fused
// runs one CTA per resident slot (cooperative launch, so all are resident)
// over balanced ranges of 16-byte vectors: pass 1 takes max |x| of each
// range (split at head boundaries) and merges it with atomicMax on the float
// bits, which order like the unsigned integers for values >= 0; a grid
// barrier; pass 2 re-reads the range (from L2 when the tensor fits there),
// derives inv from amax and writes the codes.  After every CTA has finished
// pass 2, CTA 0 turns amax into s in place and writes code vector 0 over the
// counters.  Each wait is bounded in time and records a timeout in
// g_device_error.
//
// Asymmetric mode (the same page names a zero-point beside the scale): u8
// codes.  hi = max(max x, 0) and -lo = max(max -x, 0) over the tensor or
// head (pass 1 keeps both, the second in the caller's zero-point buffer);
// w = hi - lo in IEEE double; s = RN32(w / 255), inv = RN32(min(255 / w,
// FLT_MAX)) (both 1 when w = 0); z = clamp(rint(RN32(-lo * inv)), 0, 255);
// code = clamp(rint(RN32(x * inv)) + z, 0, 255).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100.cuh"

namespace intattn {

struct QuantArgs {
  const void* x;     // [B, H, L, d] fp16 or bf16
  int8_t* out;       // [B, H, L, d]
  uint32_t* amax;    // [H] or [1]: the caller's float scale buffer, used as bits
                     // (asymmetric: max(max x, 0))
  uint32_t* nmax;    // asymmetric: the caller's zero-point buffer, holding the
                     // bits of max(max -x, 0) until the end; else null
  int64_t nvec;      // B * H * L * d / 8: 16-byte input vectors in all
  int64_t seg;       // vectors sharing one scale: L * d / 8 per head, or nvec
  int32_t H, per_head, bf16, n_scales, asym;
};

namespace quant {

constexpr int kThreads = 256;
constexpr int kVec = 8;                          // elements per 16-byte load
constexpr int kBatch = 8;                        // loads in flight per thread
constexpr int kStep = kThreads * kBatch;         // vectors per CTA and batch

constexpr unsigned kRoleGridBarrier = 4;  // role bits of a quant_fused timeout

// Programmatic dependent launch: a grid launched with programmatic stream
// serialisation may start once its predecessor has triggered (or exited);
// griddep_wait returns when the predecessor has completed and its writes
// are visible.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Waits until *ctr >= target (acquire, gpu scope).  Returns false and records
// the error after kWaitTimeoutNs.
__device__ __forceinline__ bool wait_count(const uint32_t* ctr, uint32_t target) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
  if (v >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    __nanosleep(20);
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
      atomicOr(&g_device_error, kErrTimeout | (kRoleGridBarrier << 8));
      return false;
    }
  }
}

// Vector range [lo, hi) of CTA `b` of `g`: equal shares, +-1.
__device__ __forceinline__ void cta_range(int64_t n, int64_t& lo, int64_t& hi) {
  const int64_t b = blockIdx.x, g = gridDim.x;
  lo = n / g * b + min(b, n % g);
  hi = lo + n / g + (b < n % g ? 1 : 0);
}

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

// Codes of 8 elements.  p = x * inv (fp32, rounded to nearest); adding
// 1.5 * 2^23 rounds p to an integer q with ties to even (|p| < 2^22) and
// leaves 0x400000 + q in the mantissa, so the low byte of the sum's bits is q
// as a two's complement byte.  The clamp to [-127, 127] of the definition
// never binds here: |x| <= amax gives |p| <= RN(amax * RN(127 / amax)) <=
// 127 * (1 + 2^-24), which rounds to at most 127, and with inv capped at
// FLT_MAX (amax < 127 / FLT_MAX) |p| <= amax * FLT_MAX < 127.
// RN(x * m) on a pair of floats (one packed multiply).
__device__ __forceinline__ float2 mul_rn2(float x0, float x1, float m) {
  float2 r;
  asm("{\n\t.reg .b64 xa, ma, pa;\n\t"
      "mov.b64 xa, {%2, %3};\n\t"
      "mov.b64 ma, {%4, %4};\n\t"
      "mul.rn.f32x2 pa, xa, ma;\n\t"
      "mov.b64 {%0, %1}, pa;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(x0), "f"(x1), "f"(m));
  return r;
}

// Asymmetric parameters from hi = max(max x, 0) and nl = max(max -x, 0).
struct AsymParams {
  float s, inv;
  int32_t z;
};
__device__ __forceinline__ AsymParams asym_params(uint32_t hi_bits, uint32_t nl_bits) {
  const double w = static_cast<double>(__uint_as_float(hi_bits)) + static_cast<double>(__uint_as_float(nl_bits));
  AsymParams p;
  if (w == 0.0) {
    p.s = 1.0f;
    p.inv = 1.0f;
    p.z = 0;
    return p;
  }
  p.s = __double2float_rn(__ddiv_rn(w, 255.0));
  p.inv = __double2float_rn(fmin(__ddiv_rn(255.0, w), 3.4028234663852886e38));
  const int32_t z = __float2int_rn(__fmul_rn(__uint_as_float(nl_bits), p.inv));
  p.z = min(max(z, 0), 255);
  return p;
}

// Asymmetric codes of 8 elements: rint(RN(x * inv)) as in codes8, then
// + z and the clamp to [0, 255].  zoff = 0x4B400000 - z, so that the bits of
// RN(p + 1.5 * 2^23) minus zoff are rint(p) + z.
__device__ __forceinline__ uint2 codes8_asym(uint4 v, bool bf16, float inv, int32_t zoff) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  float f[8];
  to_float8(v, bf16, f);
  uint32_t t[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = mul_rn2(f[2 * i], f[2 * i + 1], inv);
    const int32_t a = static_cast<int32_t>(__float_as_uint(__fadd_rn(p.x, kRound))) - zoff;
    const int32_t b = static_cast<int32_t>(__float_as_uint(__fadd_rn(p.y, kRound))) - zoff;
    t[2 * i] = static_cast<uint32_t>(min(max(a, 0), 255));
    t[2 * i + 1] = static_cast<uint32_t>(min(max(b, 0), 255));
  }
  return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

__device__ __forceinline__ uint2 codes8(uint4 v, bool bf16, float inv) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  float f[8];
  to_float8(v, bf16, f);
  uint32_t t[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // the adds are scalar with explicit rounding: a packed add after the
    // packed multiply was contracted into one fused operation
    const float2 p = mul_rn2(f[2 * i], f[2 * i + 1], inv);
    t[2 * i] = __float_as_uint(__fadd_rn(p.x, kRound));
    t[2 * i + 1] = __float_as_uint(__fadd_rn(p.y, kRound));
  }
  return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

// 1-D cooperative grid of at most one CTA per resident slot
__global__ void __launch_bounds__(kThreads) quant_fused_kernel(const __grid_constant__ QuantArgs a) {
  const uint4* src = static_cast<const uint4*>(a.x);
  uint2* dst = reinterpret_cast<uint2*>(a.out);
  uint32_t* arrive = reinterpret_cast<uint32_t*>(a.out);  // code bytes 0-3 until the end
  uint32_t* depart = arrive + 1;                           // code bytes 4-7
  __shared__ float red[kThreads / 32], red2[kThreads / 32];
  __shared__ int ok;
  int64_t lo0, hi;
  cta_range(a.nvec, lo0, hi);

  // pass 1: max |x| per head segment of the range (the loads start while
  // quant_zero may still run)
  bool zeroed = false;
  for (int64_t lo = lo0; lo < hi;) {
    const int64_t seg_id = lo / a.seg;
    const int64_t end = min(hi, (seg_id + 1) * a.seg);
    // max |x| as 16-bit patterns, two per word: with the sign bit cleared,
    // finite fp16 / bf16 values order like their unsigned bit patterns.
    // Asymmetric: mh takes the non-negative halves, mn the magnitudes of the
    // negative ones (a half whose sign is set counts as 0 in mh).
    uint32_t mh = 0, mn = 0;
    for (int64_t base = lo; base < end; base += kStep) {
      // all of a batch's loads are issued before any is used
      uint4 v[kBatch];
      const uint4* p = src + base + threadIdx.x;
      if (base + kStep <= end) {
#pragma unroll
        for (int it = 0; it < kBatch; ++it) v[it] = __ldg(p + it * kThreads);
      } else {
#pragma unroll
        for (int it = 0; it < kBatch; ++it)
          v[it] = base + it * kThreads + threadIdx.x < end ? __ldg(p + it * kThreads) : make_uint4(0, 0, 0, 0);
      }
      if (a.asym) {
#pragma unroll
        for (int it = 0; it < kBatch; ++it) {
          const uint32_t w4[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t sm = ((w4[c] >> 15) & 0x00010001u) * 0xFFFFu;  // each half's sign spread over the half
            mh = __vmaxu2(mh, w4[c] & ~sm);
            mn = __vmaxu2(mn, w4[c] & sm & 0x7FFF7FFFu);
          }
        }
      } else {
#pragma unroll
        for (int it = 0; it < kBatch; ++it) {
          mh = __vmaxu2(mh, v[it].x & 0x7FFF7FFFu);
          mh = __vmaxu2(mh, v[it].y & 0x7FFF7FFFu);
          mh = __vmaxu2(mh, v[it].z & 0x7FFF7FFFu);
          mh = __vmaxu2(mh, v[it].w & 0x7FFF7FFFu);
        }
      }
    }
    auto to_f = [&](uint32_t pair) {
      const uint32_t m16 = max(pair & 0xFFFFu, pair >> 16);
      return a.bf16 ? __uint_as_float(m16 << 16) : __half2float(__ushort_as_half(static_cast<unsigned short>(m16)));
    };
    float m = to_f(mh), mneg = to_f(mn);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      mneg = fmaxf(mneg, __shfl_xor_sync(0xffffffffu, mneg, o));
    }
    if ((threadIdx.x & 31) == 0) {
      red[threadIdx.x >> 5] = m;
      red2[threadIdx.x >> 5] = mneg;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < kThreads / 32; ++w) {
        m = fmaxf(m, red[w]);
        mneg = fmaxf(mneg, red2[w]);
      }
      if (!zeroed) griddep_wait();  // quant_zero has completed
      zeroed = true;
      const int e = a.per_head ? static_cast<int>(seg_id % a.H) : 0;
      atomicMax(a.amax + e, __float_as_uint(m));
      if (a.asym) atomicMax(a.nmax + e, __float_as_uint(mneg));
    }
    __syncthreads();  // red is reused by the next segment
    lo = end;
  }

  // grid barrier: every amax merged
  if (threadIdx.x == 0) {
    if (!zeroed) griddep_wait();
    __threadfence();
    atomicAdd(arrive, 1u);
    ok = wait_count(arrive, gridDim.x);
  }
  __syncthreads();
  if (!ok) return;

  // pass 2: codes, batches in the reverse order of pass 1 (the last ones
  // read are still in L1); vector 0 (the counters) is kept for the end
  uint2 first = make_uint2(0, 0);
  for (int64_t top = hi; top > lo0;) {
    const int64_t seg_id = (top - 1) / a.seg;
    const int64_t start = max(lo0, seg_id * a.seg);
    const int e = a.per_head ? static_cast<int>(seg_id % a.H) : 0;
    float inv;
    int32_t zoff = 0;
    if (a.asym) {
      const AsymParams ap = asym_params(__ldcg(a.amax + e), __ldcg(a.nmax + e));
      inv = ap.inv;
      zoff = 0x4B400000 - ap.z;
    } else {
      inv = inv_scale_of(__ldcg(a.amax + e));
    }
    auto code = [&](uint4 x) { return a.asym ? codes8_asym(x, a.bf16, inv, zoff) : codes8(x, a.bf16, inv); };
    for (int64_t base = start + (top - 1 - start) / kStep * kStep; base >= start; base -= kStep) {
      uint4 v[kBatch];
      const uint4* p = src + base + threadIdx.x;
      uint2* q = dst + base + threadIdx.x;
      if (base + kStep <= top && base != 0) {  // a full batch without vector 0
#pragma unroll
        for (int it = 0; it < kBatch; ++it) v[it] = __ldg(p + it * kThreads);
#pragma unroll
        for (int it = 0; it < kBatch; ++it) q[it * kThreads] = code(v[it]);
      } else {
#pragma unroll
        for (int it = 0; it < kBatch; ++it)
          v[it] = base + it * kThreads + threadIdx.x < top ? __ldg(p + it * kThreads) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int it = 0; it < kBatch; ++it) {
          const int64_t e = base + it * kThreads + threadIdx.x;
          if (e < top) {
            const uint2 c = code(v[it]);
            if (e == 0) first = c;
            else q[it * kThreads] = c;
          }
        }
      }
    }
    top = start;
  }

  // every CTA is past its last read of amax and of the arrival counter
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(depart, 1u);
  }
  if (blockIdx.x != 0) return;
  if (threadIdx.x == 0) ok = wait_count(depart, gridDim.x);
  __syncthreads();
  if (!ok) return;
  for (int i = threadIdx.x; i < a.n_scales; i += kThreads) {
    if (a.asym) {
      const AsymParams ap = asym_params(__ldcg(a.amax + i), __ldcg(a.nmax + i));
      a.amax[i] = __float_as_uint(ap.s);
      a.nmax[i] = static_cast<uint32_t>(ap.z);
    } else {
      a.amax[i] = __float_as_uint(scale_of(__ldcg(a.amax + i)));
    }
  }
  if (threadIdx.x == 0) dst[0] = first;  // thread 0 of CTA 0 owns vector 0
}

// one CTA: zero the amax slots (and the asymmetric second maxima) and the
// two barrier counters
__global__ void quant_zero_kernel(uint32_t* amax, uint32_t* nmax, int n, uint32_t* counters) {
  griddep_trigger();  // quant_fused waits for completion before it uses these
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    amax[i] = 0u;
    if (nmax) nmax[i] = 0u;
  }
  if (threadIdx.x < 2) counters[threadIdx.x] = 0u;
}

// one CTA, the empty tensor: every scale 1 (and every zero-point 0)
__global__ void quant_scales_kernel(uint32_t* amax, uint32_t* nmax, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    amax[i] = __float_as_uint(1.0f);
    if (nmax) nmax[i] = 0u;
  }
}

}  // namespace quant
}  // namespace intattn
