// Decode kernels: one query per (batch, head) against an int8 or a packed
// int4 KV cache.
//
// Same integer definition as the prefill path with Lq = 1 and no mask.  The
// work is an HBM stream of the K and V rows (2*Lk*d bytes per (b, h)), so it
// is split over key chunks to fill every SM, in three launches:
//   decode_qk  per (b, h, chunk): S_j = q.K_j with 16-byte vector loads and
//              dp4a; S to the workspace, chunk max to the workspace.
//   decode_z   per (b, h): m = max of the chunk maxima, Z over all Lk scores
//              (from L2), the reciprocal R; (m, R) to the workspace.
//   decode_pv  per (b, h, chunk): the u8 probabilities of this chunk from
//              (m, R); V chunk streamed with 16-byte loads, P.V by dp4a after
//              a 4x4 byte transpose; int32 partial sums to the workspace.
//              The last CTA of a (b, h) (atomic ticket) adds the partials and
//              requantises.  Integer addition is associative, so the result
//              does not depend on the order.
// The int4 cache (decode4_qk / decode_z / decode4_pv) has rows of D/2 bytes,
// byte t holding channel 2t in bits 0-3 and channel 2t+1 in bits 4-7, each a
// two's-complement value in [-8, 7].  A thread streams 16-byte pieces (32
// channels) and unpacks each 8-channel word into the biased unsigned bytes
// u = x + 8 of its even and of its odd channels (nibble ^ 8: one logic op
// per 4 channels); dp4a works on u and the bias is removed exactly:
// q.x = q.u - 8 sum(q), and sum P x = sum P u - 8 sum(P).
// Unsigned int4 codes with zero-points: a nibble c in [0, 15] stands for
// c - z; the kernels then skip the XOR (u = c) and remove z instead of 8
// (for K any per-row constant cancels in the gaps, so none is removed).
// Zero-points of the int8 cache: u8 K codes need only the dp4a operand type
// (the per-row constant q.z_k cancels in every gap); u8 V codes with
// zero-point z_v give sum P (v - z_v) = sum P v - z_v sum P, with sum P
// found by decode_z in a second sweep over the scores once R is known.
#pragma once
#include <climits>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace intattn {

struct DecodeArgs {
  const int8_t* q;   // [BH, d]
  const int8_t* k;   // [BH, Lmax, d] int8, or [BH, Lmax, d/2] packed int4
  const int8_t* v;   // same layout as k
  int8_t* out;       // [BH, d]
  int32_t* ws_s;     // [BH, ld_s]        scores (row stride ld_s = Lk rounded up to 4)
  int32_t* ws_max;   // [BH, nsplit]      chunk maxima
  int32_t* ws_part;  // [BH, nsplit, d]   partial P.V sums
  uint32_t* ws_cnt;  // [BH]              arrival tickets
  int32_t* ws_mr;    // [BH, 4]           row max, reciprocal R, sum of P (V zero-point only)
  int32_t BH, H, Lk, Lmax, nsplit, chunk, per_head, ld_s;
  int32_t k_u8, v_u8;  // K / V codes are unsigned (u8, or u4 nibbles) with zero-points
  uint32_t lut[INTATTN_MAX_CLIPS][32];  // one exp table per distinct clip threshold
  HeadParamsDev hp[INTATTN_MAX_HEADS];
};

namespace decode {

constexpr int kThreads = 256;
constexpr int kChunk = 512;    // keys per CTA, int8 cache (multiple of the rows one step covers)
// Partial-sum rows of the P.V reductions: one word of padding per row keeps
// both the per-thread writes and the per-channel reads free of bank conflicts.
constexpr int kPartStride = kThreads + 1;
constexpr int kChunk4 = 4096;  // keys per CTA, int4 cache (measured best for the 4096-key rows)

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

__device__ __forceinline__ int32_t dp4a_ss(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// signed bytes of a times unsigned bytes of b
__device__ __forceinline__ int32_t dp4a_su(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ int32_t dp4a_uu(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 8 packed int4 channels (one word) -> unsigned bytes u of the even channels
// (lo): u = x + 8 for two's complement nibbles (x8 = 0x08080808), u = c for
// unsigned ones (x8 = 0).
__device__ __forceinline__ uint32_t nib_lo(uint32_t w, uint32_t x8) { return (w & 0x0F0F0F0Fu) ^ x8; }
// The odd channels' nibbles in place: byte t holds 16 u.  Products with it
// are 16 times the unshifted ones (one op fewer than shifting down); their
// sums are divided by 16 exactly at the end.
__device__ __forceinline__ uint32_t nib_hi16(uint32_t w, uint32_t x8) { return (w & 0xF0F0F0F0u) ^ (x8 << 4); }

__device__ __forceinline__ int32_t imax32(int32_t a, int32_t b) { return a > b ? a : b; }

// Thread layout shared by both kernels: CPR = D/16 threads cover one row in
// 16-byte pieces; a thread handles 4 rows (a "quad") per step.
template <int D>
struct Layout {
  static constexpr int kCPR = D / 16;                  // 16-byte pieces per row
  static constexpr int kGroups = kThreads / kCPR;      // row quads per step
  static constexpr int kRowsPerStep = 4 * kGroups;     // 128 (d=128) or 256 (d=64)
  static_assert(kChunk % kRowsPerStep == 0, "chunk must be whole steps");
};

template <int D, bool KU8>
__global__ void __launch_bounds__(kThreads) decode_qk_kernel(const __grid_constant__ DecodeArgs a) {
  using Lt = Layout<D>;
  const int bh = blockIdx.y;
  const int sp = blockIdx.x;
  const int j0 = sp * a.chunk;
  const int j1 = min(a.Lk, j0 + a.chunk);
  const int tid = threadIdx.x;
  const int piece = tid % Lt::kCPR;
  const int grp = tid / Lt::kCPR;
  const int lane = tid & 31;

  if (sp == 0 && tid == 0) a.ws_cnt[bh] = 0u;  // ticket for decode_pv

  const uint4 qv = *reinterpret_cast<const uint4*>(a.q + static_cast<size_t>(bh) * D + piece * 16);
  const int8_t* kbase = a.k + static_cast<size_t>(bh) * a.Lmax * D + piece * 16;
  int32_t* srow = a.ws_s + static_cast<size_t>(bh) * a.ld_s;
  int32_t mx = INT_MIN;

  for (int base = j0; base < j1; base += Lt::kRowsPerStep) {
    const int r0 = base + 4 * grp;
    uint4 kv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = r0 + i;
      kv[i] = (j < j1) ? ld_stream(kbase + static_cast<size_t>(j) * D) : make_uint4(0, 0, 0, 0);
    }
    int32_t s[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int32_t acc = 0;
      if constexpr (KU8) {  // s8 q times u8 K codes
        acc = dp4a_su(qv.x, kv[i].x, acc);
        acc = dp4a_su(qv.y, kv[i].y, acc);
        acc = dp4a_su(qv.z, kv[i].z, acc);
        acc = dp4a_su(qv.w, kv[i].w, acc);
      } else {
        acc = dp4a_ss(kv[i].x, qv.x, acc);
        acc = dp4a_ss(kv[i].y, qv.y, acc);
        acc = dp4a_ss(kv[i].z, qv.z, acc);
        acc = dp4a_ss(kv[i].w, qv.w, acc);
      }
      s[i] = acc;
    }
    // reduce the CPR partial sums of each of the 4 rows (transpose-reduce)
    int32_t t0, t1;
    if (Lt::kCPR == 8) {
      const bool hi = lane & 4;
      const int32_t send0 = hi ? s[0] : s[2], send1 = hi ? s[1] : s[3];
      const int32_t keep0 = hi ? s[2] : s[0], keep1 = hi ? s[3] : s[1];
      t0 = keep0 + __shfl_xor_sync(0xffffffffu, send0, 4);
      t1 = keep1 + __shfl_xor_sync(0xffffffffu, send1, 4);
    } else {
      t0 = s[0];  // with CPR = 4 the pair (0,1)/(2,3) split happens below
      t1 = s[1];
    }
    int32_t row_val;
    int row_idx;
    if (Lt::kCPR == 8) {
      const bool b1 = lane & 2;
      const int32_t send = b1 ? t0 : t1, keep = b1 ? t1 : t0;
      int32_t u = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      u += __shfl_xor_sync(0xffffffffu, u, 1);
      row_val = u;
      row_idx = ((lane & 4) ? 2 : 0) + ((lane & 2) ? 1 : 0);
    } else {
      const bool b1 = lane & 2;
      const int32_t send0 = b1 ? s[0] : s[2], send1 = b1 ? s[1] : s[3];
      const int32_t keep0 = b1 ? s[2] : s[0], keep1 = b1 ? s[3] : s[1];
      const int32_t u0 = keep0 + __shfl_xor_sync(0xffffffffu, send0, 2);
      const int32_t u1 = keep1 + __shfl_xor_sync(0xffffffffu, send1, 2);
      const bool b0 = lane & 1;
      const int32_t send = b0 ? u0 : u1, keep = b0 ? u1 : u0;
      row_val = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      row_idx = (b1 ? 2 : 0) + (b0 ? 1 : 0);
      (void)t0;
      (void)t1;
    }
    const int j = r0 + row_idx;
    const bool writer = (Lt::kCPR == 8) ? ((lane & 1) == 0) : true;
    if (writer && j < j1) {
      srow[j] = row_val;
      mx = imax32(mx, row_val);
    }
  }
  // chunk max
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = imax32(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __shared__ int32_t red[kThreads / 32];
  if (lane == 0) red[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    int32_t r = red[0];
    for (int w = 1; w < kThreads / 32; ++w) r = imax32(r, red[w]);
    a.ws_max[static_cast<size_t>(bh) * a.nsplit + sp] = r;
  }
}

// Row max, row sum Z and reciprocal R of one (b, h): one CTA per row.
template <int D>
__global__ void __launch_bounds__(kThreads) decode_z_kernel(const __grid_constant__ DecodeArgs a) {
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int h = bh % a.H;
  const HeadParamsDev hp = a.hp[a.per_head ? h : 0];
  __shared__ uint32_t lut_s[32];
  __shared__ int32_t red[kThreads / 32];
  if (tid < 32) lut_s[tid] = a.lut[hp.lut][tid];
  int32_t m = INT_MIN;
  for (int i = 0; i < a.nsplit; ++i) m = imax32(m, __ldcg(a.ws_max + static_cast<size_t>(bh) * a.nsplit + i));
  const long long lo64 = static_cast<long long>(m) - hp.D;
  const int32_t lo = lo64 < INT_MIN ? INT_MIN : static_cast<int32_t>(lo64);
  const uint32_t Mu = static_cast<uint32_t>(hp.M);
  const uint32_t sh = static_cast<uint32_t>(hp.s);
  const uint32_t Cm = static_cast<uint32_t>(m) * Mu + (1u << (sh - 1));
  __syncthreads();
  // idx = (min(m - S, D) M + 2^(s-1)) >> s as (Cm - max(S, m - D) M) >> s in
  // wrapping 32-bit arithmetic (the true value lies in [0, 2^31))
  // rows start on 16-byte boundaries (ld_s is a multiple of 4)
  const int4* srow = reinterpret_cast<const int4*>(a.ws_s + static_cast<size_t>(bh) * a.ld_s);
  int32_t z = 0;
  const int n4 = a.Lk / 4;
  for (int i = tid; i < n4; i += kThreads) {
    const int4 s4 = __ldcg(srow + i);
    z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(imax32(s4.x, lo)) * Mu) >> sh]);
    z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(imax32(s4.y, lo)) * Mu) >> sh]);
    z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(imax32(s4.z, lo)) * Mu) >> sh]);
    z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(imax32(s4.w, lo)) * Mu) >> sh]);
  }
  for (int j = 4 * n4 + tid; j < a.Lk; j += kThreads) {
    const int32_t t = imax32(__ldcg(a.ws_s + static_cast<size_t>(bh) * a.ld_s + j), lo);
    z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(t) * Mu) >> sh]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane == 0) red[tid >> 5] = z;
  __syncthreads();
  __shared__ uint32_t R_s;
  if (tid == 0) {
    int32_t Z = 0;
    for (int w = 0; w < kThreads / 32; ++w) Z += red[w];
    const unsigned long long R =
        ((255ull << 32) + static_cast<unsigned long long>(Z >> 1)) / static_cast<unsigned long long>(Z);
    a.ws_mr[4 * bh] = m;
    a.ws_mr[4 * bh + 1] = static_cast<int32_t>(R);
    R_s = static_cast<uint32_t>(R);
  }
  if (hp.zv == 0) return;
  // V zero-point: sum_j P_j over the row, P_j from the same table as decode_pv
  __shared__ uint32_t ptab_s[32];
  __syncthreads();
  if (tid < 32)
    ptab_s[tid] = static_cast<uint32_t>((static_cast<unsigned long long>(lut_s[tid]) * R_s + (1ull << 31)) >> 32);
  __syncthreads();
  int32_t ps = 0;
  for (int j = tid; j < a.Lk; j += kThreads) {
    const int32_t t = imax32(__ldcg(a.ws_s + static_cast<size_t>(bh) * a.ld_s + j), lo);
    ps += static_cast<int32_t>(ptab_s[(Cm - static_cast<uint32_t>(t) * Mu) >> sh]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
  if (lane == 0) red[tid >> 5] = ps;
  __syncthreads();
  if (tid == 0) {
    int32_t P = 0;
    for (int w = 0; w < kThreads / 32; ++w) P += red[w];
    a.ws_mr[4 * bh + 2] = P;
  }
}

template <int D, bool VU8>
__global__ void __launch_bounds__(kThreads) decode_pv_kernel(const __grid_constant__ DecodeArgs a) {
  using Lt = Layout<D>;
  const int bh = blockIdx.y;
  const int sp = blockIdx.x;
  const int j0 = sp * a.chunk;
  const int j1 = min(a.Lk, j0 + a.chunk);
  const int tid = threadIdx.x;
  const int h = bh % a.H;
  const HeadParamsDev hp = a.hp[a.per_head ? h : 0];

  __shared__ uint32_t ptab_s[32];
  __shared__ uint32_t pk[kChunk / 4];              // u8 probabilities of this chunk
  __shared__ int32_t part[16 * kPartStride];       // per-thread partial sums, [channel][thread]
  __shared__ int last_flag;

  const int32_t m = __ldcg(a.ws_mr + 4 * bh);
  const unsigned long long R = static_cast<uint32_t>(__ldcg(a.ws_mr + 4 * bh + 1));
  if (tid < 32)
    ptab_s[tid] = static_cast<uint32_t>((static_cast<unsigned long long>(a.lut[hp.lut][tid]) * R + (1ull << 31)) >> 32);
  const long long lo64 = static_cast<long long>(m) - hp.D;
  const int32_t lo = lo64 < INT_MIN ? INT_MIN : static_cast<int32_t>(lo64);
  const uint32_t Mu = static_cast<uint32_t>(hp.M);
  const uint32_t sh = static_cast<uint32_t>(hp.s);
  const uint32_t Cm = static_cast<uint32_t>(m) * Mu + (1u << (sh - 1));
  const int32_t* srow = a.ws_s + static_cast<size_t>(bh) * a.ld_s;
  __syncthreads();

  // V rows are streamed with 16-byte loads, one step ahead of the math: the
  // first step is issued before the probabilities are computed
  const int piece = tid % Lt::kCPR;
  const int grp = tid / Lt::kCPR;
  const int8_t* vbase = a.v + static_cast<size_t>(bh) * a.Lmax * D + piece * 16;
  auto load4 = [&](int r0, uint4 (&vv)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = r0 + i;
      vv[i] = (j < j1) ? ld_stream(vbase + static_cast<size_t>(j) * D) : make_uint4(0, 0, 0, 0);
    }
  };
  uint4 cur[4];
  load4(j0 + 4 * grp, cur);

  // u8 probabilities of this chunk, 4 per word (rows past j1 get 0)
  for (int w = tid; w < a.chunk / 4; w += kThreads) {
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + 4 * w + b;
      if (j < j1) {
        const int32_t t = imax32(__ldcg(srow + j), lo);
        word |= ptab_s[(Cm - static_cast<uint32_t>(t) * Mu) >> sh] << (8 * b);
      }
    }
    pk[w] = word;
  }
  __syncthreads();

  // acc[c] over this thread's 16 columns
  int32_t acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = 0;
  for (int base = j0; base < j1; base += Lt::kRowsPerStep) {
    const int r0 = base + 4 * grp;
    const bool more = base + Lt::kRowsPerStep < j1;
    uint4 nxt[4];
    if (more) load4(r0 + Lt::kRowsPerStep, nxt);
    const uint32_t p4 = pk[(r0 - j0) >> 2];  // P of rows r0..r0+3, one byte each
    const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&cur[0]);
    const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&cur[1]);
    const uint32_t* w2 = reinterpret_cast<const uint32_t*>(&cur[2]);
    const uint32_t* w3 = reinterpret_cast<const uint32_t*>(&cur[3]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      // bytes (row i, column 4q+c) -> word c holds the 4 rows of column 4q+c
      const uint32_t ab_lo = __byte_perm(w0[q], w1[q], 0x5140);
      const uint32_t ab_hi = __byte_perm(w0[q], w1[q], 0x7362);
      const uint32_t cd_lo = __byte_perm(w2[q], w3[q], 0x5140);
      const uint32_t cd_hi = __byte_perm(w2[q], w3[q], 0x7362);
      if constexpr (VU8) {  // u8 V codes
        acc[4 * q + 0] = dp4a_uu(__byte_perm(ab_lo, cd_lo, 0x5410), p4, acc[4 * q + 0]);
        acc[4 * q + 1] = dp4a_uu(__byte_perm(ab_lo, cd_lo, 0x7632), p4, acc[4 * q + 1]);
        acc[4 * q + 2] = dp4a_uu(__byte_perm(ab_hi, cd_hi, 0x5410), p4, acc[4 * q + 2]);
        acc[4 * q + 3] = dp4a_uu(__byte_perm(ab_hi, cd_hi, 0x7632), p4, acc[4 * q + 3]);
      } else {
        acc[4 * q + 0] = dp4a_su(__byte_perm(ab_lo, cd_lo, 0x5410), p4, acc[4 * q + 0]);
        acc[4 * q + 1] = dp4a_su(__byte_perm(ab_lo, cd_lo, 0x7632), p4, acc[4 * q + 1]);
        acc[4 * q + 2] = dp4a_su(__byte_perm(ab_hi, cd_hi, 0x5410), p4, acc[4 * q + 2]);
        acc[4 * q + 3] = dp4a_su(__byte_perm(ab_hi, cd_hi, 0x7632), p4, acc[4 * q + 3]);
      }
    }
    if (more) {
#pragma unroll
      for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    }
  }
  // reduce over the row groups: column piece*16 + c
#pragma unroll
  for (int c = 0; c < 16; ++c) part[c * kPartStride + tid] = acc[c];
  __syncthreads();
  int32_t* gpart = a.ws_part + (static_cast<size_t>(bh) * a.nsplit + sp) * D;
  if (tid < D) {
    const int pc = tid / 16, c = tid % 16;
    int32_t sum = 0;
    for (int g = 0; g < Lt::kGroups; ++g) sum += part[c * kPartStride + g * Lt::kCPR + pc];
    gpart[tid] = sum;
  }
  // the last CTA of this (b, h) adds the partials and requantises
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(a.ws_cnt + bh, 1u);
    last_flag = (prev == static_cast<unsigned>(a.nsplit - 1));
  }
  __syncthreads();
  if (last_flag) {
    __threadfence();
    if (tid < D) {
      int32_t tot = 0;
      const int32_t* p0 = a.ws_part + static_cast<size_t>(bh) * a.nsplit * D + tid;
      for (int i = 0; i < a.nsplit; ++i) tot += __ldcg(p0 + static_cast<size_t>(i) * D);
      if (hp.zv != 0) tot -= hp.zv * __ldcg(a.ws_mr + 4 * bh + 2);  // sum P (v - z_v)
      const long long t = static_cast<long long>(tot) * hp.Mo + (1ll << (hp.so - 1));
      long long y = t >> hp.so;
      y = y > 127 ? 127 : (y < -127 ? -127 : y);
      a.out[static_cast<size_t>(bh) * D + tid] = static_cast<int8_t>(y);
    }
    if (tid == 0) a.ws_cnt[bh] = 0u;
  }
}


// ------------------------------------------------------------ int4 cache
// Thread layout: CPR = D/32 threads cover one row in 16-byte pieces (32
// channels); a thread handles 4 rows (a "quad") per step.
template <int D>
struct Layout4 {
  static constexpr int kCPR = D / 32;
  static constexpr int kGroups = kThreads / kCPR;
  static constexpr int kRowsPerStep = 4 * kGroups;  // 256 (d=128) or 512 (d=64)
  static_assert(kChunk4 % kRowsPerStep == 0, "chunk must be whole steps");
};

template <int D>
__global__ void __launch_bounds__(kThreads) decode4_qk_kernel(const __grid_constant__ DecodeArgs a) {
  using Lt = Layout4<D>;
  constexpr int kRowBytes = D / 2;
  const int bh = blockIdx.y;
  const int sp = blockIdx.x;
  const int j0 = sp * a.chunk;
  const int j1 = min(a.Lk, j0 + a.chunk);
  const int tid = threadIdx.x;
  const int piece = tid % Lt::kCPR;
  const int grp = tid / Lt::kCPR;
  const int lane = tid & 31;

  if (sp == 0 && tid == 0) a.ws_cnt[bh] = 0u;  // ticket for decode4_pv

  // q over this piece's 32 channels, as even / odd channel words of each
  // 8-channel group (the order the unpacked K words come in)
  const uint4 qa = *reinterpret_cast<const uint4*>(a.q + static_cast<size_t>(bh) * D + piece * 32);
  const uint4 qb = *reinterpret_cast<const uint4*>(a.q + static_cast<size_t>(bh) * D + piece * 32 + 16);
  const uint32_t qw[8] = {__byte_perm(qa.x, qa.y, 0x6420), __byte_perm(qa.x, qa.y, 0x7531),
                          __byte_perm(qa.z, qa.w, 0x6420), __byte_perm(qa.z, qa.w, 0x7531),
                          __byte_perm(qb.x, qb.y, 0x6420), __byte_perm(qb.x, qb.y, 0x7531),
                          __byte_perm(qb.z, qb.w, 0x6420), __byte_perm(qb.z, qb.w, 0x7531)};
  // unsigned codes: no bias is removed (q.z_k is the same for every key of the row)
  const uint32_t kx8 = a.k_u8 ? 0u : 0x08080808u;
  const int32_t qbias = a.k_u8 ? 0 :
      8 * dp4a_ss(qa.x, 0x01010101u, dp4a_ss(qa.y, 0x01010101u, dp4a_ss(qa.z, 0x01010101u, dp4a_ss(qa.w, 0x01010101u,
      dp4a_ss(qb.x, 0x01010101u, dp4a_ss(qb.y, 0x01010101u, dp4a_ss(qb.z, 0x01010101u, dp4a_ss(qb.w, 0x01010101u, 0))))))));
  const int8_t* kbase = a.k + static_cast<size_t>(bh) * a.Lmax * kRowBytes + piece * 16;
  int32_t* srow = a.ws_s + static_cast<size_t>(bh) * a.ld_s;
  int32_t mx = INT_MIN;

  // K rows with 16-byte loads, one step ahead of the math (two register
  // buffers in turn)
  auto load4 = [&](int r0, uint4 (&kv)[4]) {
    const int8_t* kp = kbase + static_cast<size_t>(r0) * kRowBytes;
    if (r0 + 4 <= j1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = ld_stream(kp + i * kRowBytes);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = (r0 + i < j1) ? ld_stream(kp + i * kRowBytes) : make_uint4(0, 0, 0, 0);
    }
  };
  auto quad = [&](int r0, const uint4 (&kv)[4]) {
    int32_t s[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {kv[i].x, kv[i].y, kv[i].z, kv[i].w};
      int32_t acc = -qbias, acc16 = 0;  // even channels; odd channels x 16
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        acc = dp4a_su(qw[2 * g], nib_lo(w[g], kx8), acc);
        acc16 = dp4a_su(qw[2 * g + 1], nib_hi16(w[g], kx8), acc16);
      }
      s[i] = acc + (acc16 >> 4);  // acc16 is a multiple of 16
    }
    // reduce the CPR partial sums of each of the 4 rows (transpose-reduce)
    if constexpr (Lt::kCPR == 4) {
      const bool b1 = lane & 2;
      const int32_t send0 = b1 ? s[0] : s[2], send1 = b1 ? s[1] : s[3];
      const int32_t keep0 = b1 ? s[2] : s[0], keep1 = b1 ? s[3] : s[1];
      const int32_t u0 = keep0 + __shfl_xor_sync(0xffffffffu, send0, 2);
      const int32_t u1 = keep1 + __shfl_xor_sync(0xffffffffu, send1, 2);
      const bool b0 = lane & 1;
      const int32_t send = b0 ? u0 : u1, keep = b0 ? u1 : u0;
      const int32_t row_val = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      const int j = r0 + (b1 ? 2 : 0) + (b0 ? 1 : 0);
      if (j < j1) {
        srow[j] = row_val;
        mx = imax32(mx, row_val);
      }
    } else {  // CPR == 2: lane pair (2g, 2g+1) holds rows (0,1) / (2,3) after one exchange
      const bool b0 = lane & 1;
      const int32_t send0 = b0 ? s[0] : s[2], send1 = b0 ? s[1] : s[3];
      const int32_t keep0 = b0 ? s[2] : s[0], keep1 = b0 ? s[3] : s[1];
      const int32_t u0 = keep0 + __shfl_xor_sync(0xffffffffu, send0, 1);
      const int32_t u1 = keep1 + __shfl_xor_sync(0xffffffffu, send1, 1);
      const int j = r0 + (b0 ? 2 : 0);
      if (j < j1) {
        srow[j] = u0;
        mx = imax32(mx, u0);
      }
      if (j + 1 < j1) {
        srow[j + 1] = u1;
        mx = imax32(mx, u1);
      }
    }
  };
  uint4 buf0[4], buf1[4];
  load4(j0 + 4 * grp, buf0);
  for (int base = j0; base < j1; base += 2 * Lt::kRowsPerStep) {
    const int r0 = base + 4 * grp;
    if (base + Lt::kRowsPerStep < j1) load4(r0 + Lt::kRowsPerStep, buf1);
    quad(r0, buf0);
    if (base + Lt::kRowsPerStep >= j1) break;
    if (base + 2 * Lt::kRowsPerStep < j1) load4(r0 + 2 * Lt::kRowsPerStep, buf0);
    quad(r0 + Lt::kRowsPerStep, buf1);
  }
  // chunk max
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = imax32(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __shared__ int32_t red[kThreads / 32];
  if (lane == 0) red[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    int32_t r = red[0];
    for (int w = 1; w < kThreads / 32; ++w) r = imax32(r, red[w]);
    a.ws_max[static_cast<size_t>(bh) * a.nsplit + sp] = r;
  }
}

// P.V over the int4 cache: a thread owns 16 channels (an 8-byte piece of a
// row) of 8 consecutive rows per step, so it holds 16 accumulators and keeps
// two steps of loads (128 bytes) in flight at three CTAs per SM.
template <int D>
struct LayoutPv4 {
  static constexpr int kCPR = D / 16;                // 8-byte pieces per row
  static constexpr int kGroups = kThreads / kCPR;    // row octets per step
  static constexpr int kRowsPerStep = 8 * kGroups;   // 256 (d=128) or 512 (d=64)
  static_assert(kChunk4 % kRowsPerStep == 0, "chunk must be whole steps");
};

// kOwnZ: the chunk is the whole row (nsplit == 1), so this CTA also takes
// the role of decode_z: m from the chunk maximum, Z and R from the scores it
// reads anyway to build P.  Same arithmetic as decode_z, bit for bit.
template <int D, bool kOwnZ>
__global__ void __launch_bounds__(kThreads, 4) decode4_pv_kernel(const __grid_constant__ DecodeArgs a) {
  using Lt = LayoutPv4<D>;
  constexpr int kRowBytes = D / 2;
  const int bh = blockIdx.y;
  const int sp = blockIdx.x;
  const int j0 = sp * a.chunk;
  const int j1 = min(a.Lk, j0 + a.chunk);
  const int tid = threadIdx.x;
  const int h = bh % a.H;
  const HeadParamsDev hp = a.hp[a.per_head ? h : 0];

  __shared__ uint32_t ptab_s[32];
  __shared__ uint32_t pk[kChunk4 / 4];             // u8 probabilities of this chunk
  __shared__ int32_t part[16 * kPartStride];       // per-thread partial sums, [channel][thread]
  __shared__ int last_flag;
  __shared__ int32_t zred[kThreads / 32];

  int32_t m;
  if constexpr (kOwnZ) {
    m = __ldcg(a.ws_max + bh);  // the only chunk's maximum
    if (tid < 32) ptab_s[tid] = a.lut[hp.lut][tid];  // the exp table until R is known
  } else {
    m = __ldcg(a.ws_mr + 4 * bh);
    const unsigned long long R = static_cast<uint32_t>(__ldcg(a.ws_mr + 4 * bh + 1));
    if (tid < 32)
      ptab_s[tid] = static_cast<uint32_t>((static_cast<unsigned long long>(a.lut[hp.lut][tid]) * R + (1ull << 31)) >> 32);
  }
  const long long lo64 = static_cast<long long>(m) - hp.D;
  const int32_t lo = lo64 < INT_MIN ? INT_MIN : static_cast<int32_t>(lo64);
  const uint32_t Mu = static_cast<uint32_t>(hp.M);
  const uint32_t sh = static_cast<uint32_t>(hp.s);
  const uint32_t Cm = static_cast<uint32_t>(m) * Mu + (1u << (sh - 1));
  const int32_t* srow = a.ws_s + static_cast<size_t>(bh) * a.ld_s;
  __syncthreads();

  // V rows streamed with 8-byte loads, one step ahead of the math (two
  // register buffers in turn)
  const int piece = tid % Lt::kCPR;
  const int grp = tid / Lt::kCPR;
  const int8_t* vbase = a.v + static_cast<size_t>(bh) * a.Lmax * kRowBytes + piece * 8;
  auto load8 = [&](int r0, uint2 (&vv)[8]) {
    const int8_t* p = vbase + static_cast<size_t>(r0) * kRowBytes;
    if (r0 + 8 <= j1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) vv[i] = ld_stream8(p + i * kRowBytes);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) vv[i] = (r0 + i < j1) ? ld_stream8(p + i * kRowBytes) : make_uint2(0, 0);
    }
  };
  uint2 buf0[8], buf1[8];
  load8(j0 + 8 * grp, buf0);  // in flight while the probabilities are built

  if constexpr (kOwnZ) {
    // indices first (bytes of pk) and Z = sum of their table entries; then R,
    // the probability table, and the indices turned into probabilities
    int32_t z = 0;
    for (int w = tid; w < a.chunk / 4; w += kThreads) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = j0 + 4 * w + b;
        if (j < j1) {
          const uint32_t idx = (Cm - static_cast<uint32_t>(imax32(__ldcg(srow + j), lo)) * Mu) >> sh;
          z += static_cast<int32_t>(ptab_s[idx]);
          word |= idx << (8 * b);
        } else {
          word |= 32u << (8 * b);  // past the row: probability 0 (entry 32 below)
        }
      }
      pk[w] = word;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if ((tid & 31) == 0) zred[tid >> 5] = z;
    __syncthreads();
    if (tid < 32) {  // each lane turns its own table entry into a probability
      int32_t Z = 0;
      for (int i = 0; i < kThreads / 32; ++i) Z += zred[i];
      const unsigned long long R =
          ((255ull << 32) + static_cast<unsigned long long>(Z >> 1)) / static_cast<unsigned long long>(Z);
      ptab_s[tid] = static_cast<uint32_t>((static_cast<unsigned long long>(ptab_s[tid]) * R + (1ull << 31)) >> 32);
    }
    __syncthreads();
    for (int w = tid; w < a.chunk / 4; w += kThreads) {
      const uint32_t x = pk[w];
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t idx = (x >> (8 * b)) & 0xFFu;
        word |= (idx < 32u ? ptab_s[idx] : 0u) << (8 * b);
      }
      pk[w] = word;
    }
  } else {
    for (int w = tid; w < a.chunk / 4; w += kThreads) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = j0 + 4 * w + b;
        if (j < j1) {
          const int32_t t = imax32(__ldcg(srow + j), lo);
          word |= ptab_s[(Cm - static_cast<uint32_t>(t) * Mu) >> sh] << (8 * b);
        }
      }
      pk[w] = word;
    }
  }
  __syncthreads();

  // acc[4u + c], u = 2g + e: channel 8g + 2c + e of this thread's 16
  int32_t acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = 0;
  int32_t psum = 0;  // sum of this thread's P: the bias correction
  const uint32_t vx8 = a.v_u8 ? 0u : 0x08080808u;
  const int32_t vbias = a.v_u8 ? hp.zv : 8;  // what each V code is offset by
  auto octet = [&](int r0, const uint2 (&cur)[8]) {
#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {  // the two row quads of the octet
      const uint32_t p4 = pk[((r0 - j0) >> 2) + hq];  // P of 4 rows, one byte each (0 past j1)
      psum = dp4a_uu(p4, 0x01010101u, psum);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t y0 = g ? cur[4 * hq + 0].y : cur[4 * hq + 0].x;
        const uint32_t y1 = g ? cur[4 * hq + 1].y : cur[4 * hq + 1].x;
        const uint32_t y2 = g ? cur[4 * hq + 2].y : cur[4 * hq + 2].x;
        const uint32_t y3 = g ? cur[4 * hq + 3].y : cur[4 * hq + 3].x;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // e = 1: the odd channels, 16 x biased (accumulators divided by 16 at the end)
          const uint32_t x0 = e ? nib_hi16(y0, vx8) : nib_lo(y0, vx8);
          const uint32_t x1 = e ? nib_hi16(y1, vx8) : nib_lo(y1, vx8);
          const uint32_t x2 = e ? nib_hi16(y2, vx8) : nib_lo(y2, vx8);
          const uint32_t x3 = e ? nib_hi16(y3, vx8) : nib_lo(y3, vx8);
          // bytes (row i, column c) -> word c holds the 4 rows of column c
          const uint32_t ab_lo = __byte_perm(x0, x1, 0x5140);
          const uint32_t ab_hi = __byte_perm(x0, x1, 0x7362);
          const uint32_t cd_lo = __byte_perm(x2, x3, 0x5140);
          const uint32_t cd_hi = __byte_perm(x2, x3, 0x7362);
          const int o = 4 * (2 * g + e);
          acc[o + 0] = dp4a_uu(__byte_perm(ab_lo, cd_lo, 0x5410), p4, acc[o + 0]);
          acc[o + 1] = dp4a_uu(__byte_perm(ab_lo, cd_lo, 0x7632), p4, acc[o + 1]);
          acc[o + 2] = dp4a_uu(__byte_perm(ab_hi, cd_hi, 0x5410), p4, acc[o + 2]);
          acc[o + 3] = dp4a_uu(__byte_perm(ab_hi, cd_hi, 0x7632), p4, acc[o + 3]);
        }
      }
    }
  };
  for (int base = j0; base < j1; base += 2 * Lt::kRowsPerStep) {
    const int r0 = base + 8 * grp;
    if (base + Lt::kRowsPerStep < j1) load8(r0 + Lt::kRowsPerStep, buf1);
    octet(r0, buf0);
    if (base + Lt::kRowsPerStep >= j1) break;
    if (base + 2 * Lt::kRowsPerStep < j1) load8(r0 + 2 * Lt::kRowsPerStep, buf0);
    octet(r0 + Lt::kRowsPerStep, buf1);
  }
  // per-thread sums by channel, bias removed; then reduce over the row groups
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    const int g = s >> 3, e = (s >> 2) & 1, c = s & 3;
    part[(8 * g + 2 * c + e) * kPartStride + tid] = (e ? (acc[s] >> 4) : acc[s]) - vbias * psum;  // acc >= 0
  }
  __syncthreads();
  int32_t* gpart = a.ws_part + (static_cast<size_t>(bh) * a.nsplit + sp) * D;
  if (tid < D) {
    const int pc = tid / 16, c = tid % 16;
    int32_t sum = 0;
    for (int g = 0; g < Lt::kGroups; ++g) sum += part[c * kPartStride + g * Lt::kCPR + pc];
    gpart[tid] = sum;
  }
  // the last CTA of this (b, h) adds the partials and requantises
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(a.ws_cnt + bh, 1u);
    last_flag = (prev == static_cast<unsigned>(a.nsplit - 1));
  }
  __syncthreads();
  if (last_flag) {
    __threadfence();
    if (tid < D) {
      int32_t tot = 0;
      const int32_t* p0 = a.ws_part + static_cast<size_t>(bh) * a.nsplit * D + tid;
      for (int i = 0; i < a.nsplit; ++i) tot += __ldcg(p0 + static_cast<size_t>(i) * D);
      const long long t = static_cast<long long>(tot) * hp.Mo + (1ll << (hp.so - 1));
      long long y = t >> hp.so;
      y = y > 127 ? 127 : (y < -127 ? -127 : y);
      a.out[static_cast<size_t>(bh) * D + tid] = static_cast<int8_t>(y);
    }
    if (tid == 0) a.ws_cnt[bh] = 0u;
  }
}

}  // namespace decode
}  // namespace intattn
