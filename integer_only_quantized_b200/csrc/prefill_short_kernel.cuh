// Short-row prefill kernel (rows of at most 256 keys) of the fully-integer
// attention forward for sm_100a: the same definition as prefill_kernel.cuh
// (IntAttention, arXiv 2511.21513, "Methodology" items 2-3), with the scores
// of a whole row tile materialised in tensor memory instead of recomputed.
//
// The final row max fixes every LUT index and the final Z fixes every
// probability, so three sweeps over a row's keys remain (A: max, B: Z,
// C: P and P.V).  With at most two key tiles, both S tiles of a 128-row
// tile (256 TMEM columns) stay resident from pass A to pass C: Q.K^T runs
// once per key tile, and the softmax warps never wait for the tensor core
// between passes.  Pass C releases each S buffer right after reading it, and
// the tensor core computes the next tile's scores for that key tile before
// this tile's P.V of the same key tile, so the next tile's scores are ready
// when pass C ends.
// (Kept in shared memory instead, one byte of index code per key costs more
// to pack and unpack, at 2 cycles per byte permute, than recomputing the
// index from the resident scores, at 3 full-rate instructions per key.)
// Zero-points of K and V as in prefill_kernel.cuh: u8 K needs nothing but
// the MMA's operand type; a V zero-point adds one correction P tile per
// query tile (the four column groups' shares of sum_j P_j).
// Work unit and schedule: one (batch, head, 128-query tile), persistent CTAs
// in snake order over the tiles sorted longest first (causal).
// Warp roles (22 warps):
//   warps 0-15  IndexSoftmax, one team: warp w reads TMEM lane quadrant w % 4
//               (query rows 32(w%4) .. +31, one row per thread) and columns
//               32(w/4) .. +31 of every S tile.  The four threads of a row
//               are in the four warps of one quadrant, which combine their
//               partial max and Z through shared memory and a named barrier
//               of their own (one per quadrant), so quadrants never wait on
//               each other.
//   warp 16     TMA producer (one issuing lane per ring slot, one for Q).
//   warp 17     TMEM allocator and MMA issuer.
//   warps 18-21 epilogue: O -> requantised int8 rows.
#pragma once
#include <cuda.h>
#include <climits>
#include <cstdint>

#include "common.cuh"
#include "prefill_kernel.cuh"
#include "sm100.cuh"

namespace intattn {
namespace shortrow {

using prefill::exact_R;
using prefill::fma2_rz;
using prefill::fma_rz_sat;
using prefill::imax;
using prefill::kBM;
using prefill::kBN;
using prefill::pack2;
using prefill::pack4;
using prefill::requant_byte;
using prefill::Tile;
using prefill::tile_index;
using prefill::tile_of;

constexpr int kMaxKeyTiles = 2;              // rows of at most 256 keys: both S tiles resident
constexpr int kMaxKeys = kMaxKeyTiles * kBN;
constexpr int kSoftWarps = 16;
constexpr int kColGroups = 4;                // column groups of an S tile
constexpr int kCols = kBN / kColGroups;      // 32 S columns per thread and tile
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kEpiWarp0 = 18;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);  // 704
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S of key tile j in [128 j, 128 j + 128)
constexpr uint32_t kColO = 256;  // O accumulators: d columns each (two for d = 64)
constexpr uint32_t kColP = 384;  // four P buffers of 32 columns (128 u8 keys each)
constexpr int kPBufs = 4;
constexpr uint32_t kNbQuad0 = 1;  // named barriers 1..4: the four warps of one TMEM lane quadrant

enum Role : unsigned { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3, kRoleEpilogue = 4 };

enum Bar : int {
  kBarQFull = 0,    // [2]
  kBarQEmpty = 2,   // [2]  every Q.K^T that read that Q buffer is done
  kBarSFull = 4,    // [2]  per key tile j: S_j written
  kBarSEmpty = 6,   // [2]  all 16 softmax warps have read S_j for the last time
  kBarPFull = 8,    // [4]
  kBarPEmpty = 12,  // [4]
  kBarOFull = 16,   // [2]
  kBarOEmpty = 18,  // [2]
  kBarDrain = 20,
  kBarKvFull = 21,  // [stages], then kv_empty[stages]
};

// ZV: the kernel instance that supports a V zero-point (the correction tile
// and the sums of P); the other instance is the plain int8 kernel.
template <int D, bool ZV = false>
struct Cfg {
  static constexpr int kStages = (D == 64) ? 8 : 6;
  static constexpr int kOBufs = (D == 64) ? 2 : 1;
  static_assert(kColO + kOBufs * D <= kColP, "O buffers overlap the P buffers");
  static constexpr uint32_t kTileBytes = kBN * D;
  static constexpr uint32_t kQBytes = kBM * D;
  static constexpr uint32_t kSwizzle = (D == 128) ? 2u : 4u;
  static constexpr uint32_t kSBO = 8 * D;
  static constexpr int kNumBars = kBarKvFull + 2 * kStages;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kOffQ + 2 * kQBytes;
  // the V zero-point correction tile [32 keys][D] s8, laid out like a V tile:
  // rows 8 g: -1, rows 8 g + 1 .. 8 g + 4: -128 (g = column group), else 0
  static constexpr uint32_t kOffCorr = kOffKV + kStages * kTileBytes;
  static constexpr int kCorrGroup = 8;
  // probability table, four copies [b][33][kBM] u32 holding P << 8b
  static constexpr uint32_t kPtabBytes = 33 * kBM * 4;
  static constexpr uint32_t kOffPtab = kOffCorr + (ZV ? 32 * D : 0);
  static constexpr uint32_t kOffRed = kOffPtab + 4 * kPtabBytes;             // [2][kColGroups][kBM] int32
  static constexpr uint32_t kOffLut = kOffRed + 2 * kColGroups * kBM * 4;
  static constexpr uint32_t kOffHp = kOffLut + INTATTN_MAX_CLIPS * 32 * 4;   // head parameters
  static constexpr uint32_t kOffBars = kOffHp + INTATTN_MAX_HEADS * sizeof(HeadParamsDev);
  static constexpr uint32_t kOffTmem = kOffBars + kNumBars * 8;
  static constexpr uint32_t kUsed = kOffTmem + 16;
  // one CTA per SM (each CTA allocates all 512 TMEM columns)
  static constexpr uint32_t kSmemBytes = (kUsed + 1024 > 120 * 1024) ? kUsed + 1024 : 120 * 1024;
};

// The order in which the tensor core consumes K/V tiles (and the producer
// loads them) for one CTA with tiles t = 0, 1, ...:
//   Q.K^T of tile 0, key tiles 0 .. n0-1;
//   then for each t: for j = 0, 1: Q.K^T of tile t+1, key tile j (if it
//   has one), then P.V of tile t, key tile j (if it has one).
// `begin(t)` is called before the first Q.K^T of tile t; `qk(t, tile, j)`
// and `pv(t, tile, j)` in the order above; any of them returns false to
// stop the walk.
template <typename BEGIN, typename QK, typename PV>
__device__ __forceinline__ void walk_schedule(const PrefillArgs& a, BEGIN&& begin, QK&& qk, PV&& pv) {
  int L = tile_index(0, blockIdx.x, gridDim.x);
  if (L >= a.n_tiles) return;
  Tile T = tile_of(a, L);
  if (!begin(0, T)) return;
  for (int j = 0; j < T.nkt; ++j)
    if (!qk(0, T, j)) return;
  for (int t = 0;; ++t) {
    const int Ln = tile_index(t + 1, blockIdx.x, gridDim.x);
    const bool more = Ln < a.n_tiles;
    Tile Tn{};
    if (more) {
      Tn = tile_of(a, Ln);
      if (!begin(t + 1, Tn)) return;
    }
    for (int j = 0; j < kMaxKeyTiles; ++j) {
      if (more && j < Tn.nkt && !qk(t + 1, Tn, j)) return;
      if (j < T.nkt && !pv(t, T, j)) return;
    }
    if (!more) return;
    T = Tn;
  }
}

template <int D, bool ZV>
__global__ void __launch_bounds__(kThreads, 1) prefill_short_kernel(const __grid_constant__ PrefillArgs args) {
  using C = Cfg<D, ZV>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sKV = s_base + C::kOffKV;
  uint32_t* ptab = reinterpret_cast<uint32_t*>(smem + C::kOffPtab);
  int32_t* red = reinterpret_cast<int32_t*>(smem + C::kOffRed);
  uint32_t* lut_s = reinterpret_cast<uint32_t*>(smem + C::kOffLut);
  HeadParamsDev* hp_s = reinterpret_cast<HeadParamsDev*>(smem + C::kOffHp);
  const uint32_t bars = s_base + C::kOffBars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  auto bar_kv_full = [&](int i) { return bar(kBarKvFull + i); };
  auto bar_kv_empty = [&](int i) { return bar(kBarKvFull + C::kStages + i); };
  auto sQ = [&](uint32_t i) { return s_base + C::kOffQ + i * C::kQBytes; };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (args.status != nullptr && *args.status != 0u) return;  // parameters out of range: no output

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarQFull + i), 1);
      mbar_init(bar(kBarQEmpty + i), 1);
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), kSoftWarps);
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(bar(kBarPFull + i), kSoftWarps);
      mbar_init(bar(kBarPEmpty + i), 1);
    }
    for (int i = 0; i < C::kOBufs; ++i) {
      mbar_init(bar(kBarOFull + i), 1);
      mbar_init(bar(kBarOEmpty + i), kEpiWarps);
    }
    mbar_init(bar(kBarDrain), 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar_kv_full(i), 1);
      mbar_init(bar_kv_empty(i), 1);
    }
    mbar_fence_init();
  }
  for (int i = tid; i < args.n_luts * 32; i += blockDim.x) lut_s[i] = args.lut[i >> 5][i & 31];
  // head parameters in shared memory: a dynamically indexed kernel argument
  // is a constant-bank load that can miss
  for (int i = tid; i < (args.per_head ? args.H : 1); i += blockDim.x) hp_s[i] = args.hp_dev ? args.hp_dev[i] : args.hp[i];
  if constexpr (ZV) {
    uint32_t* corr = reinterpret_cast<uint32_t*>(smem + C::kOffCorr);
    for (int i = tid; i < 8 * D; i += blockDim.x) {
      const int key = (4 * i) / D % C::kCorrGroup;
      corr[i] = key == 0 ? 0xFFFFFFFFu : (key <= 4 ? 0x80808080u : 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kSoftWarps) {
    // ======================= IndexSoftmax warps =======================
    const int quad = warp & 3;
    const int g = warp >> 2;                 // column group: columns 32g .. 32g+31 of each S tile
    const int r = quad * 32 + lane;          // query row within the tile == TMEM lane
    const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t trow = tlane + kColS + g * kCols;
    const uint32_t prow = smem_u32(ptab) + 4u * r;  // row k of copy b at prow + 512 k + b kPtabBytes
    if (g == 0)
      for (int b = 0; b < 4; ++b) ptab[b * (C::kPtabBytes / 4) + r] = 0u;  // row 0 (masked keys) stays 0
    bool ok = true;
    uint32_t sfill[kMaxKeyTiles] = {0, 0};  // fills of each S buffer consumed so far
    uint32_t pc = 0;                        // P tiles written so far
    auto quad_sync = [&](bool mine) { return bar_red_and(kNbQuad0 + quad, 128, mine); };
    auto arrive_warp = [&](uint32_t b) {
      __syncwarp();
      if (lane == 0) mbar_arrive(b);
    };
    constexpr uint32_t kMaskedBits = 0x4B000000u;
    const unsigned long long k32x2 = pack2(32.0f), k2p23x2 = pack2(8388608.0f);

    int L = tile_index(0, blockIdx.x, gridDim.x);
    Tile T = L < args.n_tiles ? tile_of(args, L) : Tile{};
    for (int it = 0; L < args.n_tiles; ++it) {
      const int Ln = tile_index(it + 1, blockIdx.x, gridDim.x);
      const Tile Tn = Ln < args.n_tiles ? tile_of(args, Ln) : Tile{};
      const HeadParamsDev hp = hp_s[args.per_head ? T.h : 0];
      const uint32_t* lut_h = lut_s + 32 * hp.lut;
      const int32_t lut_lane =
          __float_as_int(lane == 0 ? 0.f : __int2float_rn(static_cast<int32_t>(lut_h[lane - 1])));
      const int off = args.Lk - args.Lq;
      const int key_lim = args.causal ? min(args.Lk, T.q0 + r + off + 1) : args.Lk;
      // valid keys of this thread's 32 columns of key tile j: a prefix
      auto nvalid = [&](int j) { return min(max(key_lim - (j * kBN + g * kCols), 0), kCols); };
      // a warp whose 32 rows are all past the last query row skips the
      // arithmetic (its four quadrant warps skip together); it still takes
      // part in every barrier and hand-off
      const bool rows_live = T.q0 + quad * 32 < args.Lq;
      // work of this warp on key tile j: live rows and at least one valid key
      auto live = [&](int j) { return rows_live && __any_sync(0xffffffffu, nvalid(j) > 0); };

      // ---- pass A: row max over valid keys ----
      int32_t m = INT_MIN;
#pragma unroll
      for (int j = 0; j < kMaxKeyTiles; ++j) {
        if (j >= T.nkt || !ok) break;
        if (!mbar_wait_warp(bar(kBarSFull + j), sfill[j] & 1u, kRoleSoftmax)) { ok = false; break; }
        tc_fence_after();
        if (!live(j)) continue;
        const int nv = nvalid(j);
        uint32_t v[32];
        tmem_ld32(trow + j * kBN, v);
        tmem_wait_ld();
        if (nv == kCols) {
          int32_t m4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            m4[0] = __vimax3_s32(m4[0], static_cast<int32_t>(v[k + 0]), static_cast<int32_t>(v[k + 1]));
            m4[1] = __vimax3_s32(m4[1], static_cast<int32_t>(v[k + 2]), static_cast<int32_t>(v[k + 3]));
            m4[2] = __vimax3_s32(m4[2], static_cast<int32_t>(v[k + 4]), static_cast<int32_t>(v[k + 5]));
            m4[3] = __vimax3_s32(m4[3], static_cast<int32_t>(v[k + 6]), static_cast<int32_t>(v[k + 7]));
          }
          m = imax(m, imax(imax(m4[0], m4[1]), imax(m4[2], m4[3])));
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) m = imax(m, k < nv ? static_cast<int32_t>(v[k]) : INT_MIN);
        }
      }
      red[g * kBM + r] = m;
      // also carries a failure of the previous tile's pass C to the whole quadrant
      if (!quad_sync(ok)) { ok = false; break; }
      m = imax(imax(red[r], red[kBM + r]), imax(red[2 * kBM + r], red[3 * kBM + r]));

      // LUT index code of a score on the FP32 pipe (see prefill_kernel.cuh):
      // the bits 0x4B000000 + k, k = idx + 1 for idx <= 30 and k = 32 for a
      // clipped gap; the low 5 bits are the shuffle lane, k the table row.
      // The second multiply-add of two scores is one packed instruction.
      const uint32_t Cx = 0x4B000000u + static_cast<uint32_t>(m);
      const float Mf = __int2float_rn(hp.M);
      const float Ms32 = Mf * __uint_as_float(static_cast<uint32_t>(127 - 5 - hp.s) << 23);
      const float c1 = (1.5f - Mf * __uint_as_float(static_cast<uint32_t>(127 + 23 - hp.s) << 23)) * 0.03125f;
      auto idx_bits2 = [&](uint32_t s0, uint32_t s1, uint32_t& b0, uint32_t& b1) {
        const float y0 = fma_rz_sat(__uint_as_float(Cx - s0), Ms32, c1);
        const float y1 = fma_rz_sat(__uint_as_float(Cx - s1), Ms32, c1);
        float k0, k1;
        fma2_rz(y0, y1, k32x2, k2p23x2, k0, k1);
        b0 = __float_as_uint(k0);
        b1 = __float_as_uint(k1);
      };
      // codes of 4 scores v[o .. o+3] of this thread's columns, masked past nv
      auto codes4 = [&](const uint32_t* v, int o, int nv, bool full, uint32_t (&kb)[4]) {
        idx_bits2(v[0], v[1], kb[0], kb[1]);
        idx_bits2(v[2], v[3], kb[2], kb[3]);
        if (!full) {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            if (o + b >= nv) kb[b] = kMaskedBits;
        }
      };

      // ---- pass B: Z = sum of pseudo-exponentials ----
      float z4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < kMaxKeyTiles; ++j) {
        if (j >= T.nkt || !ok) break;
        if (!live(j)) continue;
        const int nv = nvalid(j);
        const bool full = nv == kCols;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[16];
          tmem_ld16(trow + j * kBN + 16 * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t kb[4];
            codes4(v + 4 * q, 16 * h + 4 * q, nv, full, kb);
#pragma unroll
            for (int b = 0; b < 4; ++b)
              z4[b] += __int_as_float(__shfl_sync(0xffffffffu, lut_lane, static_cast<int>(kb[b])));
          }
        }
      }
      // exact: each partial is below 2^24
      red[(kColGroups + g) * kBM + r] = __float2int_rn((z4[0] + z4[1]) + (z4[2] + z4[3]));
      if (!quad_sync(ok)) { ok = false; break; }
      if (rows_live) {
        // rows past the last query row of a live warp read zero-filled Q:
        // all their scores are 0, so Z >= 2^15 there too
        const int32_t Z = (red[kColGroups * kBM + r] + red[(kColGroups + 1) * kBM + r]) +
                          (red[(kColGroups + 2) * kBM + r] + red[(kColGroups + 3) * kBM + r]);
        const unsigned long long R = exact_R(Z);
#pragma unroll
        for (int i = g * 8; i < g * 8 + 8; ++i) {
          const uint32_t P = static_cast<uint32_t>((static_cast<unsigned long long>(lut_h[i]) * R + (1ull << 31)) >> 32);
#pragma unroll
          for (int b = 0; b < 4; ++b) ptab[b * (C::kPtabBytes / 4) + (i + 1) * kBM + r] = P << (8 * b);
        }
      }
      if (!quad_sync(ok)) { ok = false; break; }  // this quadrant's table rows are complete

      // ---- pass C: P into TMEM for the P.V MMAs; each S buffer released after its last read ----
      const bool corr = ZV && hp.zv != 0;  // V zero-point: sum this thread's P bytes
      uint32_t psum = 0;
#pragma unroll
      for (int j = 0; j < kMaxKeyTiles; ++j) {
        if (j >= T.nkt || !ok) break;
        const uint32_t pi = pc + j;
        const uint32_t pb = pi & (kPBufs - 1);
        if (!mbar_wait_warp(bar(kBarPEmpty + pb), ((pi / kPBufs) & 1) ^ 1, kRoleSoftmax)) { ok = false; break; }
        uint32_t pw[8];
        if (live(j)) {
          const int nv = nvalid(j);
          const bool full = nv == kCols;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t v[16];
            tmem_ld16(trow + j * kBN + 16 * h, v);
            tmem_wait_ld();
            if (h == 1) {  // the last read of S_j
              tc_fence_before();
              arrive_warp(bar(kBarSEmpty + j));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t kb[4], p[4];
              codes4(v + 4 * q, 16 * h + 4 * q, nv, full, kb);
#pragma unroll
              for (int b = 0; b < 4; ++b) p[b] = lds_u32(kb[b] * 512u + prow + b * C::kPtabBytes);
              pw[4 * h + q] = (p[0] + p[1]) + (p[2] + p[3]);
            }
          }
        } else {
          tc_fence_before();
          arrive_warp(bar(kBarSEmpty + j));
#pragma unroll
          for (int q = 0; q < 8; ++q) pw[q] = 0u;  // masked columns: the P.V reads zeros there
        }
        if (rows_live) {  // rows past the last query row: their P is never used
          if (corr) {
#pragma unroll
            for (int q = 0; q < 8; ++q) psum = __dp4a(pw[q], 0x01010101u, psum);
          }
          tmem_st8(tlane + kColP + pb * 32 + g * (kCols / 4), pw);
          tmem_wait_st();
        }
        tc_fence_before();
        arrive_warp(bar(kBarPFull + pb));
        ++sfill[j];
      }
      if (corr && ok) {
        // the correction tile, P index pc + nkt: column group g's share in keys 8 g ..
        const uint32_t pi = pc + T.nkt;
        const uint32_t pb = pi & (kPBufs - 1);
        if (!mbar_wait_warp(bar(kBarPEmpty + pb), ((pi / kPBufs) & 1) ^ 1, kRoleSoftmax)) {
          ok = false;
        } else {
          if (rows_live) {
            uint32_t w0, w1;
            zv_correction_bytes(hp.zv * static_cast<int32_t>(psum), w0, w1);
            tmem_st2(tlane + kColP + pb * 32 + g * (C::kCorrGroup / 4), w0, w1);
            tmem_wait_st();
          }
          tc_fence_before();
          arrive_warp(bar(kBarPFull + pb));
        }
      }
      pc += T.nkt + (corr ? 1 : 0);
      L = Ln;
      T = Tn;
    }
  } else if (warp >= kEpiWarp0) {
    // ============================ epilogue ============================
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    for (int it = 0;; ++it) {
      const int L = tile_index(it, blockIdx.x, gridDim.x);
      if (L >= args.n_tiles) break;
      const Tile T = tile_of(args, L);
      const HeadParamsDev hp = hp_s[args.per_head ? T.h : 0];
      const int ob = it % C::kOBufs;
      if (!mbar_wait_warp(bar(kBarOFull + ob), (it / C::kOBufs) & 1, kRoleEpilogue)) break;
      tc_fence_after();
      const int row = T.q0 + r;
      uint4* o = reinterpret_cast<uint4*>(args.out + (static_cast<size_t>(T.bh) * args.Lq + row) * D);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(tlane + kColO + ob * D + 16 * c, v);
        tmem_wait_ld();
        if (c == D / 16 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarOEmpty + ob));
        }
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          w[q] = pack4(requant_byte(static_cast<int32_t>(v[4 * q + 0]), hp.Mo, hp.so),
                       requant_byte(static_cast<int32_t>(v[4 * q + 1]), hp.Mo, hp.so),
                       requant_byte(static_cast<int32_t>(v[4 * q + 2]), hp.Mo, hp.so),
                       requant_byte(static_cast<int32_t>(v[4 * q + 3]), hp.Mo, hp.so));
        if (row < args.Lq) o[c] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else if (warp == kProducerWarp) {
    // ============================ TMA producer ============================
    // Lane s < kStages owns ring slot s and issues every K/V load that lands
    // there (load n goes to slot n % kStages), walking the tensor core's
    // consumption order; lane kQLane issues the Q loads.
    constexpr int kQLane = 31;
    static_assert(C::kStages <= kQLane, "one lane per ring slot");
    if (lane == 0) {
      tma_prefetch_desc(&args.tm_q);
      tma_prefetch_desc(&args.tm_k);
      tma_prefetch_desc(&args.tm_v);
    }
    __syncwarp();
    if (lane < C::kStages) {
      const uint32_t slot = static_cast<uint32_t>(lane);
      const uint32_t dst = sKV + slot * C::kTileBytes;
      uint32_t n = 0, mine = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* tm, int j, int bh) {
        if (n % C::kStages == slot) {
          if (!mbar_wait(bar_kv_empty(slot), (mine & 1) ^ 1, kRoleProducer)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(bar_kv_full(slot), C::kTileBytes);
            tma_load_3d(dst, tm, bar_kv_full(slot), 0, j * kBN, bh);
            ++mine;
          }
        }
        ++n;
        return ok;
      };
      walk_schedule(
          args, [](int, const Tile&) { return true; },
          [&](int, const Tile& T, int j) { return load(&args.tm_k, j, T.bh); },
          [&](int, const Tile& T, int j) { return load(&args.tm_v, j, T.bh); });
      if (mine > 0) mbar_wait(bar_kv_full(slot), (mine - 1) & 1, kRoleProducer);
    } else if (lane == kQLane) {
      uint32_t nq = 0;
      for (int it = 0;; ++it) {
        const int L = tile_index(it, blockIdx.x, gridDim.x);
        if (L >= args.n_tiles) break;
        const Tile T = tile_of(args, L);
        const uint32_t qb = nq & 1;
        if (!mbar_wait(bar(kBarQEmpty + qb), ((nq >> 1) & 1) ^ 1, kRoleProducer)) break;
        mbar_arrive_expect_tx(bar(kBarQFull + qb), C::kQBytes);
        tma_load_3d(sQ(qb), &args.tm_q, bar(kBarQFull + qb), 0, T.q0, T.bh);
        ++nq;
      }
      for (uint32_t i = 0; i < 2 && i < nq; ++i) {
        const uint32_t last = nq - 1 - i;
        mbar_wait(bar(kBarQFull + (last & 1)), (last >> 1) & 1, kRoleProducer);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ============================= MMA issuer =============================
    const uint32_t idesc_qk = idesc_i8(kBM, kBN, 1, args.k_u8 ? 0u : 1u, 0);  // s8 x (s8 | u8), K-major B
    const uint32_t idesc_pv = idesc_i8(kBM, D, 0, args.v_u8 ? 0u : 1u, 1);    // u8 x (s8 | u8), N-major B
    constexpr uint32_t idesc_corr = idesc_i8(kBM, D, 0, 1, 1);                // u8 x s8: the correction tile
    const uint64_t kv_desc0 = smem_desc(sKV, 16, C::kSBO, C::kSwizzle);
    const uint64_t corr_desc = smem_desc(s_base + C::kOffCorr, 16, C::kSBO, C::kSwizzle);
    constexpr uint32_t kSlotDesc = C::kTileBytes >> 4;
    uint32_t slot = 0, kv_par = 0;
    uint32_t sfill0 = 0, sfill1 = 0;  // fills of each S buffer issued (two scalars: j is not a constant here)
    uint32_t pc = 0;                  // P tiles consumed
    auto next_slot = [&]() {
      if (++slot == static_cast<uint32_t>(C::kStages)) {
        slot = 0;
        kv_par ^= 1;
      }
    };
    auto begin = [&](int t, const Tile&) {
      return mbar_wait_warp(bar(kBarQFull + (t & 1)), (t >> 1) & 1, kRoleMma);
    };
    auto qk = [&](int t, const Tile& T, int j) {
      // S_j free: all softmax warps have read the previous fill of this buffer
      const uint32_t fills = j ? sfill1 : sfill0;
      if (!mbar_wait2_warp(bar(kBarSEmpty + j), (fills & 1) ^ 1, bar_kv_full(slot), kv_par, kRoleMma))
        return false;
      tc_fence_after();
      const uint32_t qb = static_cast<uint32_t>(t & 1);
      const uint64_t q_desc = smem_desc(sQ(qb), 16, C::kSBO, C::kSwizzle);
      const uint64_t k_desc = kv_desc0 + slot * kSlotDesc;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + kColS + j * kBN, q_desc + 2 * kk, k_desc + 2 * kk, idesc_qk, kk > 0);
        mma_commit(bar_kv_empty(slot));
        mma_commit(bar(kBarSFull + j));
        if (j == T.nkt - 1) mma_commit(bar(kBarQEmpty + qb));  // the tile's last read of its Q buffer
      }
      __syncwarp();
      next_slot();
      if (j) ++sfill1;
      else ++sfill0;
      return true;
    };
    auto pv = [&](int t, const Tile& T, int j) {
      const int ob = t % C::kOBufs;
      if (j == 0 && !mbar_wait_warp(bar(kBarOEmpty + ob), ((t / C::kOBufs) & 1) ^ 1, kRoleMma)) return false;
      const uint32_t pb = pc & (kPBufs - 1);
      if (!mbar_wait2_warp(bar(kBarPFull + pb), (pc / kPBufs) & 1, bar_kv_full(slot), kv_par, kRoleMma))
        return false;
      tc_fence_after();
      const uint64_t v_desc = kv_desc0 + slot * kSlotDesc;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kBN / 32; ++kk)
          mma_i8_ts(tmem + kColO + ob * D, tmem + kColP + pb * 32 + kk * 8, v_desc + ((32u * D * kk) >> 4),
                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_kv_empty(slot));
        mma_commit(bar(kBarPEmpty + pb));
      }
      __syncwarp();
      next_slot();
      ++pc;
      if (j == T.nkt - 1) {
        if (ZV && hp_s[args.per_head ? T.h : 0].zv != 0) {
          // O -= z_v sum_j P_j through the correction tile
          const uint32_t cb = pc & (kPBufs - 1);
          if (!mbar_wait_warp(bar(kBarPFull + cb), (pc / kPBufs) & 1, kRoleMma)) return false;
          tc_fence_after();
          if (elect_one()) {
            mma_i8_ts(tmem + kColO + ob * D, tmem + kColP + cb * 32, corr_desc, idesc_corr, 1u);
            mma_commit(bar(kBarPEmpty + cb));
          }
          __syncwarp();
          ++pc;
        }
        mma_commit_elect(bar(kBarOFull + ob));
      }
      return true;
    };
    walk_schedule(args, begin, qk, pv);
    // every MMA this warp issued is complete before TMEM is released
    mma_commit_elect(bar(kBarDrain));
    mbar_wait_warp(bar(kBarDrain), 0, kRoleMma);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace shortrow
}  // namespace intattn
