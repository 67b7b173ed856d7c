// Integer GELU over int8 codes: the IndexSoftmax machinery (an index by
// integer multiply and shift, a 32-entry integer table, a requantising
// multiply and shift) applied to GELU(x) = x * Phi(x).  The euno.news summary
// "[Paper] IntAttention：全整数注意力流水线用于高效边缘推理", section
// 局限性与未来工作, names GELU as the next operator for the method; the
// definition is this library's reading:
//
//   idx = clamp(16 + floor(q * M / 2^s), 0, 31)     gate point nearest s_x q
//   y   = q * G[idx]                                G = 2^15 Phi on [-c, c],
//                                                   G[0] = 0, G[31] = 2^15
//   out = clamp(floor((y * Mo + 2^(so-1)) / 2^so), -127, 127)
//
// The output depends on the code alone, so each CTA first evaluates the
// definition for all 256 codes into a shared-memory table (one copy per bank:
// entry u of lane l at word u * 32 + l, so a warp's lookups never conflict),
// then streams 16-byte vectors: one table read per element.  The first batch
// of loads is issued before the table is built.
#pragma once
#include <cstdint>

namespace intattn {

struct GeluArgs {
  const int8_t* x;
  int8_t* y;
  int64_t n;        // elements
  int32_t M, s;     // index multiplier and shift
  int32_t Mo, so;   // requant multiplier and shift
  int32_t gate[32];
};

namespace gelu {

constexpr int kThreads = 256;  // the table build assumes 256 (one code per thread)
constexpr int kBatch = 8;  // 16-byte loads in flight per thread

// The definition for one code.
__device__ __forceinline__ uint32_t code_of(int q, const GeluArgs& a) {
  int64_t idx = 16 + ((static_cast<int64_t>(q) * a.M) >> a.s);
  idx = idx < 0 ? 0 : (idx > 31 ? 31 : idx);
  const int64_t y = static_cast<int64_t>(q) * a.gate[idx];
  int64_t t = (y * a.Mo + (int64_t{1} << (a.so - 1))) >> a.so;
  t = t < -127 ? -127 : (t > 127 ? 127 : t);
  return static_cast<uint32_t>(t) & 0xFFu;
}

__device__ __forceinline__ uint4 ld_stream16(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Four codes of word w through the table; lane4 = 4 * lane.
__device__ __forceinline__ uint32_t map4(uint32_t w, const uint8_t* tab, uint32_t lane4) {
  // byte k of w is u; its entry for this lane sits at byte (u * 32 + lane) * 4
  const uint32_t b0 = *reinterpret_cast<const uint32_t*>(tab + (((w << 7) & 0x7F80u) | lane4));
  const uint32_t b1 = *reinterpret_cast<const uint32_t*>(tab + (((w >> 1) & 0x7F80u) | lane4));
  const uint32_t b2 = *reinterpret_cast<const uint32_t*>(tab + (((w >> 9) & 0x7F80u) | lane4));
  const uint32_t b3 = *reinterpret_cast<const uint32_t*>(tab + (((w >> 17) & 0x7F80u) | lane4));
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// 1-D grid of at most one wave; grid-stride over 16-byte vectors.
__global__ void __launch_bounds__(kThreads) gelu_kernel(const __grid_constant__ GeluArgs a) {
  __shared__ __align__(16) uint32_t tab[256 * 32];
  const uint4* src = reinterpret_cast<const uint4*>(a.x);
  uint4* dst = reinterpret_cast<uint4*>(a.y);
  const int64_t nvec = a.n >> 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads * kBatch;
  int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kBatch;

  uint4 v[kBatch];
#pragma unroll
  for (int it = 0; it < kBatch; ++it) {
    const int64_t e = base + it * kThreads + threadIdx.x;
    v[it] = e < nvec ? ld_stream16(src + e) : make_uint4(0, 0, 0, 0);
  }
  // table: thread t evaluates code (int8)(t) once; then each warp writes 512
  // contiguous bytes per store (16-byte stores of one entry's copies), which
  // touches every bank once
  __shared__ uint32_t codes[256];
  codes[threadIdx.x] = code_of(static_cast<int8_t>(threadIdx.x), a);
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w = 4u * threadIdx.x + 1024u * k;  // first of 4 words, all of entry w / 32
    const uint32_t out = codes[w >> 5];
    *reinterpret_cast<uint4*>(tab + w) = make_uint4(out, out, out, out);
  }
  __syncthreads();

  const uint8_t* tb = reinterpret_cast<const uint8_t*>(tab);
  const uint32_t lane4 = (threadIdx.x & 31u) * 4u;
  while (base < nvec) {
#pragma unroll
    for (int it = 0; it < kBatch; ++it) {
      const int64_t e = base + it * kThreads + threadIdx.x;
      if (e < nvec)
        dst[e] = make_uint4(map4(v[it].x, tb, lane4), map4(v[it].y, tb, lane4), map4(v[it].z, tb, lane4),
                            map4(v[it].w, tb, lane4));
    }
    base += stride;
#pragma unroll
    for (int it = 0; it < kBatch; ++it) {
      const int64_t e = base + it * kThreads + threadIdx.x;
      v[it] = e < nvec ? ld_stream16(src + e) : make_uint4(0, 0, 0, 0);
    }
  }
  // the last n % 16 elements, one per thread of CTA 0
  if (blockIdx.x == 0) {
    const int64_t i = (nvec << 4) + threadIdx.x;
    if (threadIdx.x < 16 && i < a.n) {
      const uint32_t u = static_cast<uint8_t>(a.x[i]);
      a.y[i] = static_cast<int8_t>(tab[u * 32 + (threadIdx.x & 31u)]);
    }
  }
}

}  // namespace gelu
}  // namespace intattn
