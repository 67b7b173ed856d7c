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
// gap_kernel (rows too long to keep in shared memory): one CTA per sampled row.  Scores fit in 22 bits (|S| <= 128^2 d < 2^21),
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


// The same statistic with each row's scores computed once: a CTA takes
// kRowsMax sampled rows of one (b, h) (rows blockIdx.x * kRowsMax ..), reads
// every K row once for all of them (dp4a against each query row), keeps the
// scores in shared memory [rows][n_max], and runs the radix selects of its
// rows side by side there, a group of 128 threads per row.  Dynamic shared memory: nrows * n_max * 4 bytes plus the query
// rows; the host uses this kernel while that fits.
constexpr int kRowsMax = 4;
constexpr int kRowsThreads = 512;  // 16 warps: the K loads of one CTA per SM need them in flight

__global__ void __launch_bounds__(kRowsThreads) gap_rows_kernel(const __grid_constant__ CalibArgs a, int nrows_cta,
                                                            int nsampled) {
  extern __shared__ __align__(16) int32_t sc[];  // [nrows_cta][n_stride] scores
  __shared__ uint32_t qs[kRowsMax][32];          // query rows, d / 4 words each
  __shared__ uint32_t rhist[kRowsMax][256];
  __shared__ int32_t red[kRowsThreads / 32];
  __shared__ uint32_t rprefix[kRowsMax], rrank[kRowsMax];
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * nrows_cta;          // first sampled-row number of this CTA
  const int nr = min(nrows_cta, nsampled - r0);   // rows of this CTA
  const int words = a.d / 4;
  auto row_of = [&](int r) { return (r0 + r + 1) * a.stride - 1; };
  auto nvalid = [&](int i) { return a.causal ? min(a.Lk, i + a.Lk - a.Lq + 1) : a.Lk; };
  const int n_max = nvalid(row_of(nr - 1));       // the last row sees the most keys
  const int n_stride = (n_max + 3) & ~3;
  for (int t = threadIdx.x; t < nr * words; t += kRowsThreads) {
    const int r = t / words, w = t - r * words;
    qs[r][w] = reinterpret_cast<const uint32_t*>(a.q + (static_cast<size_t>(bh) * a.Lq + row_of(r)) * a.d)[w];
  }
  __syncthreads();
  const int8_t* kb = a.k + static_cast<size_t>(bh) * a.Lk * a.d;
  // every K row once, against each query row of the CTA
  for (int j = threadIdx.x; j < n_max; j += kRowsThreads) {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + static_cast<size_t>(j) * a.d);
    int acc[kRowsMax] = {0, 0, 0, 0};
    for (int w = 0; w < words / 4; ++w) {
      const uint4 kv = __ldg(kr + w);
#pragma unroll
      for (int r = 0; r < kRowsMax; ++r) {
        if (r < nr) {
          acc[r] = __dp4a(static_cast<int>(kv.x), static_cast<int>(qs[r][4 * w]), acc[r]);
          acc[r] = __dp4a(static_cast<int>(kv.y), static_cast<int>(qs[r][4 * w + 1]), acc[r]);
          acc[r] = __dp4a(static_cast<int>(kv.z), static_cast<int>(qs[r][4 * w + 2]), acc[r]);
          acc[r] = __dp4a(static_cast<int>(kv.w), static_cast<int>(qs[r][4 * w + 3]), acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsMax; ++r)
      if (r < nr) sc[r * n_stride + j] = acc[r];
  }
  __syncthreads();
  // the radix select of the CTA's rows side by side: row g by threads
  // g * kGroup .. g * kGroup + kGroup - 1; the digit of each pass found by
  // the group's first warp (8 bins per lane, counts summed from the top)
  constexpr int kGroup = kRowsThreads / kRowsMax;  // 128 threads per row
  const int g = threadIdx.x / kGroup, gt = threadIdx.x % kGroup;
  const bool live = g < nr;
  const int n = live ? nvalid(row_of(g)) : 0;
  const int32_t* srow = sc + g * n_stride;
  int32_t m = INT_MIN;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = 16 - 8 * pass;  // digit: bits shift .. shift + 7 of u = S + 2^23
    for (int b = gt; b < 256; b += kGroup) rhist[g][b] = 0u;
    if (pass == 0 && gt == 0) {
      rprefix[g] = 0u;
      rrank[g] = static_cast<uint32_t>(min(a.keep, max(n, 1)));
    }
    __syncthreads();
    const uint32_t pre = rprefix[g];
    for (int j = gt; j < n; j += kGroup) {
      const int32_t v = srow[j];
      if (pass == 0) m = max(m, v);
      const uint32_t u = static_cast<uint32_t>(v + (1 << 23));
      if (pass == 0 || (u >> (shift + 8)) == pre) atomicAdd(&rhist[g][(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (live && gt < 32) {
      // lane l holds bins 255 - 8 l .. 248 - 8 l (from the top)
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        c[t] = rhist[g][255 - 8 * gt - t];
        tot += c[t];
      }
      uint32_t incl = tot;  // inclusive sum over lanes 0 .. gt (higher bins first)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (gt >= o) incl += y;
      }
      const uint32_t before = incl - tot;  // counts in higher bins than this lane's
      const uint32_t rk = rrank[g];
      // the lane whose bins take the cumulative count from below rk to >= rk
      const bool here = before < rk && incl >= rk;
      const unsigned who = __ballot_sync(0xffffffffu, here);
      if (here) {
        uint32_t r = rk - before, digit = 255 - 8 * gt;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (c[t] >= r) break;
          r -= c[t];
          --digit;
        }
        rprefix[g] = (pre << 8) | digit;
        rrank[g] = r;
      }
      if (who == 0u && gt == 0) {  // fewer keys than the rank cannot happen (rk <= n); keep digit 0
        rprefix[g] = pre << 8;
        rrank[g] = 1u;
      }
    }
    __syncthreads();
  }
  // row max over the group's two warps, then the gap
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (live && gt == 0) {
    int32_t mm = INT_MIN;
    for (int w = 0; w < kGroup / 32; ++w) mm = max(mm, red[g * (kGroup / 32) + w]);
    atomicMax(a.G + bh, mm - (static_cast<int32_t>(rprefix[g]) - (1 << 23)));
  }
}

}  // namespace calib
}  // namespace intattn
