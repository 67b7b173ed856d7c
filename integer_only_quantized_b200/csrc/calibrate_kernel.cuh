// Adaptive clip threshold: the integer statistic behind it, on the device.
//
// The summary pages (sections 概览 / Overview and 局限性与未来工作 /
// Limitations & Future Work) describe the clip as sparsity-aware and name an
// adaptive threshold as future work.  The rule (see intattn.h,
// intattn_calibrate_clip): for every sampled query row i of a (batch, head),
// G_i = m_i - S_i,(K), the gap from the row max to the K-th largest score
// over the valid keys (to the smallest with fewer than K); G = max over the
// sampled rows.  The host turns G into the threshold.
//
// One CTA per sampled row.  Scores fit in 22 bits (|S| <= 128^2 d < 2^21),
// so u = S + 2^23 is a 24-bit key ordered like S; the K-th largest u is
// found by a radix select of three 8-bit digits, most significant first: a
// 256-bin histogram of the keys that match the digits chosen so far, then
// the digit at which the count from the top reaches the remaining rank.
// Each pass recomputes the row's scores (dp4a over d / 4 words), so no score
// buffer is needed whatever Lk is.
#pragma once
#include <climits>
#include <cstdint>

namespace intattn {

struct CalibArgs {
  const int8_t* q;  // [B, H, Lq, d]
  const int8_t* k;  // [B, H, Lk, d]
  int32_t* G;       // [B*H], zeroed by the caller; atomicMax of each row's gap
  int32_t Lq, Lk, d, causal, keep, stride;
};

namespace calib {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) gap_kernel(const __grid_constant__ CalibArgs a) {
  __shared__ uint32_t qs[32];       // the query row, d / 4 words (d <= 128)
  __shared__ uint32_t hist[256];
  __shared__ int32_t red[kThreads / 32];
  __shared__ uint32_t prefix, rank;  // digits chosen so far; rank still to find among them
  const int bh = blockIdx.y;
  const int i = (blockIdx.x + 1) * a.stride - 1;  // sampled row
  const int n = a.causal ? min(a.Lk, i + a.Lk - a.Lq + 1) : a.Lk;  // valid keys
  const int words = a.d / 4;
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(a.q + (static_cast<size_t>(bh) * a.Lq + i) * a.d);
  if (threadIdx.x < words) qs[threadIdx.x] = qrow[threadIdx.x];
  __syncthreads();
  const int8_t* kb = a.k + static_cast<size_t>(bh) * a.Lk * a.d;
  auto score = [&](int j) {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + static_cast<size_t>(j) * a.d);
    int acc = 0;
    for (int w = 0; w < words / 4; ++w) {
      const uint4 kv = __ldg(kr + w);
      acc = __dp4a(static_cast<int>(kv.x), static_cast<int>(qs[4 * w]), acc);
      acc = __dp4a(static_cast<int>(kv.y), static_cast<int>(qs[4 * w + 1]), acc);
      acc = __dp4a(static_cast<int>(kv.z), static_cast<int>(qs[4 * w + 2]), acc);
      acc = __dp4a(static_cast<int>(kv.w), static_cast<int>(qs[4 * w + 3]), acc);
    }
    return acc;
  };
  int32_t m = INT_MIN;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = 16 - 8 * pass;  // digit: bits shift .. shift + 7 of u
    for (int b = threadIdx.x; b < 256; b += kThreads) hist[b] = 0u;
    if (pass == 0 && threadIdx.x == 0) {
      prefix = 0u;
      rank = static_cast<uint32_t>(min(a.keep, n));
    }
    __syncthreads();
    const uint32_t pre = prefix;
    for (int j = threadIdx.x; j < n; j += kThreads) {
      const int32_t s = score(j);
      if (pass == 0) m = max(m, s);
      const uint32_t u = static_cast<uint32_t>(s + (1 << 23));
      // keys whose higher digits equal the ones chosen so far
      if (pass == 0 || (u >> (shift + 8)) == pre) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t r = rank, digit = 255;
      for (;; --digit) {  // from the top: the digit where the count reaches the rank
        if (hist[digit] >= r || digit == 0) break;
        r -= hist[digit];
      }
      prefix = (pre << 8) | digit;
      rank = r;
    }
    __syncthreads();
  }
  // row max
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kThreads / 32; ++w) m = max(m, red[w]);
    const int32_t kth = static_cast<int32_t>(prefix) - (1 << 23);
    atomicMax(a.G + bh, m - kth);
  }
}

}  // namespace calib
}  // namespace intattn
