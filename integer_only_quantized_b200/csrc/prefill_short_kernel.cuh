// Short-row prefill kernel (rows of at most 512 keys) of the fully-integer
// attention forward for sm_100a: the same definition as prefill_kernel.cuh
// (IntAttention, arXiv 2511.21513, "Methodology" items 2-3), with the LUT
// index codes of a row materialised in registers instead of recomputing the
// scores for the last sweep.
//
// The final row max fixes every LUT index and the final Z fixes every
// probability, so three sweeps over a row's keys remain (A: max, B: Z,
// C: P and P.V).  What changes for short rows:
//   * pass B keeps the index code of every score it visits (one byte per
//     key, 32 keys of each of at most 4 key tiles per thread: at most 32
//     registers), so pass C reads codes from registers and needs neither a
//     third Q.K^T nor the S tiles;
//   * with at most 2 key tiles (<= 256 keys) both S tiles stay resident in
//     TMEM from pass A to pass B: Q.K^T runs once per key tile in total;
//   * the next tile's first Q.K^T goes to the tensor core ahead of this
//     tile's P.V, as soon as pass B has released the S buffers, so S is ready
//     when the softmax warps finish pass C.
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

using prefill::fma_rz_sat;
using prefill::imax;
using prefill::kBM;
using prefill::kBN;
using prefill::pack4;
using prefill::requant_byte;
using prefill::Tile;
using prefill::tile_index;
using prefill::tile_of;

constexpr int kMaxKeyTiles = 4;              // rows of at most 512 keys
constexpr int kMaxKeys = kMaxKeyTiles * kBN;
constexpr int kResidentTiles = 2;            // key tiles whose S stays in TMEM from pass A to B
constexpr int kSoftWarps = 16;
constexpr int kColGroups = 4;                // column groups of an S tile
constexpr int kCols = kBN / kColGroups;      // 32 S columns per thread and tile
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kEpiWarp0 = 18;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);  // 704
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // two S buffers: [0,128) and [128,256)
constexpr uint32_t kColO = 256;  // O accumulators: d columns each (two for d = 64)
constexpr uint32_t kColP = 384;  // four P buffers of 32 columns (128 u8 keys each)
constexpr int kPBufs = 4;
constexpr uint32_t kNbQuad0 = 1;  // named barriers 1..4: the four warps of one TMEM lane quadrant

enum Role : unsigned { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3, kRoleEpilogue = 4 };

enum Bar : int {
  kBarQFull = 0,    // [2]
  kBarQEmpty = 2,   // [2]  every Q.K^T that read that Q buffer is done
  kBarSFull = 4,    // [2]
  kBarSEmpty = 6,   // [2]  all 16 softmax warps are done with the S tile
  kBarPFull = 8,    // [4]
  kBarPEmpty = 12,  // [4]
  kBarOFull = 16,   // [2]
  kBarOEmpty = 18,  // [2]
  kBarDrain = 20,
  kBarKvFull = 21,  // [stages], then kv_empty[stages]
};

template <int D>
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
  static constexpr uint32_t kOffPtab = kOffKV + kStages * kTileBytes;      // [33][kBM] u32
  static constexpr uint32_t kOffRed = kOffPtab + 33 * kBM * 4;            // [2][kColGroups][kBM] int32
  static constexpr uint32_t kOffLut = kOffRed + 2 * kColGroups * kBM * 4;
  static constexpr uint32_t kOffBars = kOffLut + INTATTN_MAX_CLIPS * 32 * 4;
  static constexpr uint32_t kOffTmem = kOffBars + kNumBars * 8;
  static constexpr uint32_t kUsed = kOffTmem + 16;
  // one CTA per SM (each CTA allocates all 512 TMEM columns)
  static constexpr uint32_t kSmemBytes = (kUsed + 1024 > 120 * 1024) ? kUsed + 1024 : 120 * 1024;
};

// The order in which the tensor core consumes K/V tiles (and the producer
// loads them) for one CTA: for tile t with n key tiles,
//   Q.K^T of its first min(n, 2) key tiles (pass A), then P.V of tile t-1,
//   then Q.K^T of its other key tiles (pass A), then, when n > 2, Q.K^T of
//   all n key tiles again (pass B); after the last tile, its P.V.
// `qk(tile, j)` and `pv(tile, j)` are called in that order; they return false
// to stop the walk.
template <typename QK, typename PV, typename BEGIN>
__device__ __forceinline__ void walk_schedule(const PrefillArgs& a, BEGIN&& begin, QK&& qk, PV&& pv) {
  Tile prev{};
  int it = 0;
  for (;; ++it) {
    const int L = tile_index(it, blockIdx.x, gridDim.x);
    if (L >= a.n_tiles) break;
    const Tile T = tile_of(a, L);
    if (!begin(it, T)) return;
    const int lead = T.nkt < kResidentTiles ? T.nkt : kResidentTiles;
    for (int j = 0; j < lead; ++j)
      if (!qk(it, T, j)) return;
    if (it > 0)
      for (int j = 0; j < prev.nkt; ++j)
        if (!pv(it - 1, prev, j)) return;
    for (int j = lead; j < T.nkt; ++j)
      if (!qk(it, T, j)) return;
    if (T.nkt > kResidentTiles)
      for (int j = 0; j < T.nkt; ++j)
        if (!qk(it, T, j)) return;
    prev = T;
  }
  if (it > 0)
    for (int j = 0; j < prev.nkt; ++j)
      if (!pv(it - 1, prev, j)) return;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_short_kernel(const __grid_constant__ PrefillArgs args) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sKV = s_base + C::kOffKV;
  uint32_t* ptab = reinterpret_cast<uint32_t*>(smem + C::kOffPtab);
  int32_t* red = reinterpret_cast<int32_t*>(smem + C::kOffRed);
  uint32_t* lut_s = reinterpret_cast<uint32_t*>(smem + C::kOffLut);
  const uint32_t bars = s_base + C::kOffBars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  auto bar_kv_full = [&](int i) { return bar(kBarKvFull + i); };
  auto bar_kv_empty = [&](int i) { return bar(kBarKvFull + C::kStages + i); };
  auto sQ = [&](uint32_t i) { return s_base + C::kOffQ + i * C::kQBytes; };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

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
    const uint32_t trow = tlane + g * kCols;
    const uint32_t prow = smem_u32(ptab) + 4u * r;  // row k of the table at prow + 512 k
    if (g == 0) ptab[r] = 0u;                        // table row 0 (masked keys) stays 0
    bool ok = true;
    uint32_t sc = 0;  // S fills consumed so far (the MMA warp counts the same way)
    uint32_t pc = 0;  // P tiles written so far
    auto quad_sync = [&](bool mine) { return bar_red_and(kNbQuad0 + quad, 128, mine); };
    auto arrive_warp = [&](uint32_t b) {
      __syncwarp();
      if (lane == 0) mbar_arrive(b);
    };
    auto s_buf = [&](uint32_t fill) { return kColS + (fill & 1u) * kBN; };
    auto wait_s = [&](uint32_t fill) {
      return mbar_wait_warp(bar(kBarSFull + (fill & 1u)), (fill >> 1) & 1u, kRoleSoftmax);
    };
    auto release_s = [&](uint32_t fill) {
      tc_fence_before();
      arrive_warp(bar(kBarSEmpty + (fill & 1u)));
    };
    constexpr uint32_t kMaskedBits = 0x4B000000u;

    for (int it = 0;; ++it) {
      const int L = tile_index(it, blockIdx.x, gridDim.x);
      if (L >= args.n_tiles) break;
      const Tile T = tile_of(args, L);
      const HeadParamsDev hp = args.hp[args.per_head ? T.h : 0];
      const uint32_t* lut_h = lut_s + 32 * hp.lut;
      const int32_t lut_lane =
          __float_as_int(lane == 0 ? 0.f : __int2float_rn(static_cast<int32_t>(lut_h[lane - 1])));
      const int off = args.Lk - args.Lq;
      const int key_lim = args.causal ? min(args.Lk, T.q0 + r + off + 1) : args.Lk;
      // valid keys of this thread's 32 columns of key tile j: a prefix
      auto nvalid = [&](int j) { return min(max(key_lim - (j * kBN + g * kCols), 0), kCols); };
      const bool resident = T.nkt <= kResidentTiles;

      // ---- pass A: row max over valid keys ----
      int32_t m = INT_MIN;
#pragma unroll
      for (int j = 0; j < kMaxKeyTiles; ++j) {
        if (j >= T.nkt || !ok) break;
        const uint32_t fill = sc + j;
        if (!wait_s(fill)) { ok = false; break; }
        tc_fence_after();
        const int nv = nvalid(j);
        uint32_t v[32];
        tmem_ld32(trow + s_buf(fill), v);
        tmem_wait_ld();
        if (!resident) release_s(fill);
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
      if (!resident) sc += T.nkt;
      red[g * kBM + r] = m;
      // also carries a failure of the previous tile's pass C to the whole quadrant
      if (!quad_sync(ok)) { ok = false; break; }
      m = imax(imax(red[r], red[kBM + r]), imax(red[2 * kBM + r], red[3 * kBM + r]));

      // LUT index code of a score on the FP32 pipe (see prefill_kernel.cuh):
      // the bits 0x4B000000 + k, k = idx + 1 for idx <= 30 and k = 32 for a
      // clipped gap; the low byte is k, the low 5 bits the shuffle lane.
      const uint32_t Cx = 0x4B000000u + static_cast<uint32_t>(m);
      const float Mf = __int2float_rn(hp.M);
      const float Ms32 = Mf * __uint_as_float(static_cast<uint32_t>(127 - 5 - hp.s) << 23);
      const float c1 = (1.5f - Mf * __uint_as_float(static_cast<uint32_t>(127 + 23 - hp.s) << 23)) * 0.03125f;
      auto idx_bits = [&](uint32_t sv) {
        const float y = fma_rz_sat(__uint_as_float(Cx - sv), Ms32, c1);
        return __float_as_uint(__fmaf_rz(y, 32.0f, 8388608.0f));
      };

      // ---- pass B: Z, and the code of every key kept in registers ----
      uint32_t codes[kMaxKeyTiles][8];
      float zf = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxKeyTiles; ++j) {
        if (j >= T.nkt || !ok) break;
        const uint32_t fill = sc + j;
        if (!resident) {
          if (!wait_s(fill)) { ok = false; break; }
          tc_fence_after();
        }
        const int nv = nvalid(j);
        float z4[4] = {0.f, 0.f, 0.f, 0.f};
        // two halves of 16 columns: fewer scores live next to the codes
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[16];
          tmem_ld16(trow + s_buf(fill) + 16 * h, v);
          tmem_wait_ld();
          if (h == 1) release_s(fill);
          const bool full = nv == kCols;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t kb[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const int k = 4 * q + b;
              kb[b] = (full || 16 * h + k < nv) ? idx_bits(v[k]) : kMaskedBits;
              z4[b] += __int_as_float(__shfl_sync(0xffffffffu, lut_lane, static_cast<int>(kb[b])));
            }
            codes[j][4 * h + q] = pack4(kb[0], kb[1], kb[2], kb[3]);
          }
        }
        zf += (z4[0] + z4[1]) + (z4[2] + z4[3]);  // exact: below 2^24
      }
      sc += T.nkt;
      red[(kColGroups + g) * kBM + r] = __float2int_rn(zf);
      if (!quad_sync(ok)) { ok = false; break; }
      const int32_t Z = (red[kColGroups * kBM + r] + red[(kColGroups + 1) * kBM + r]) +
                        (red[(kColGroups + 2) * kBM + r] + red[(kColGroups + 3) * kBM + r]);
      {
        // R = floor(N / Z), N = 255 2^32 + floor(Z/2): the double quotient is
        // within one unit of R; one integer step makes it exact
        const unsigned long long N = (255ull << 32) + static_cast<unsigned long long>(Z >> 1);
        const unsigned long long Zu = static_cast<unsigned long long>(Z);
        unsigned long long R =
            static_cast<unsigned long long>(__ddiv_rn(static_cast<double>(N), static_cast<double>(Z)));
        if (R * Zu > N) --R;
        else if ((R + 1) * Zu <= N) ++R;
#pragma unroll
        for (int i = g * 8; i < g * 8 + 8; ++i)
          ptab[(i + 1) * kBM + r] =
              static_cast<uint32_t>((static_cast<unsigned long long>(lut_h[i]) * R + (1ull << 31)) >> 32);
      }
      if (!quad_sync(ok)) { ok = false; break; }  // this quadrant's table rows are complete

      // ---- pass C: P from the codes into TMEM for the P.V MMAs ----
#pragma unroll
      for (int j = 0; j < kMaxKeyTiles; ++j) {
        if (j >= T.nkt || !ok) break;
        const uint32_t pi = pc + j;
        const uint32_t pb = pi & (kPBufs - 1);
        if (!mbar_wait_warp(bar(kBarPEmpty + pb), ((pi / kPBufs) & 1) ^ 1, kRoleSoftmax)) { ok = false; break; }
        uint32_t pw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t w = codes[j][q];
          uint32_t p[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) p[b] = lds_u32(__byte_perm(w, 0u, 0x4440u + b) * 512u + prow);
          pw[q] = pack4(p[0], p[1], p[2], p[3]);
        }
        tmem_st8(tlane + kColP + pb * 32 + g * (kCols / 4), pw);
        tmem_wait_st();
        tc_fence_before();
        arrive_warp(bar(kBarPFull + pb));
      }
      pc += T.nkt;
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
      const HeadParamsDev hp = args.hp[args.per_head ? T.h : 0];
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
    constexpr uint32_t idesc_qk = idesc_i8(kBM, kBN, 1, 1, 0);  // s8 x s8, K-major B
    constexpr uint32_t idesc_pv = idesc_i8(kBM, D, 0, 1, 1);    // u8 x s8, N-major B
    const uint64_t kv_desc0 = smem_desc(sKV, 16, C::kSBO, C::kSwizzle);
    constexpr uint32_t kSlotDesc = C::kTileBytes >> 4;
    uint32_t slot = 0, kv_par = 0;
    uint32_t sc = 0;   // S fills issued
    uint32_t pc = 0;   // P tiles consumed
    int qk_left = 0;   // Q.K^T of the current tile still to issue
    uint32_t qb = 0;
    auto next_slot = [&]() {
      if (++slot == static_cast<uint32_t>(C::kStages)) {
        slot = 0;
        kv_par ^= 1;
      }
    };
    auto begin = [&](int it, const Tile& T) {
      qb = static_cast<uint32_t>(it & 1);
      qk_left = T.nkt > kResidentTiles ? 2 * T.nkt : T.nkt;
      return mbar_wait_warp(bar(kBarQFull + qb), (it >> 1) & 1, kRoleMma);
    };
    auto qk = [&](int, const Tile&, int) {
      const uint32_t buf = sc & 1;
      if (!mbar_wait2_warp(bar(kBarSEmpty + buf), ((sc >> 1) & 1) ^ 1, bar_kv_full(slot), kv_par, kRoleMma))
        return false;
      tc_fence_after();
      const uint64_t q_desc = smem_desc(sQ(qb), 16, C::kSBO, C::kSwizzle);
      const uint64_t k_desc = kv_desc0 + slot * kSlotDesc;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + kColS + buf * kBN, q_desc + 2 * kk, k_desc + 2 * kk, idesc_qk, kk > 0);
        mma_commit(bar_kv_empty(slot));
        mma_commit(bar(kBarSFull + buf));
        if (qk_left == 1) mma_commit(bar(kBarQEmpty + qb));  // the tile's last read of its Q buffer
      }
      __syncwarp();
      next_slot();
      ++sc;
      --qk_left;
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
        if (j == T.nkt - 1) mma_commit(bar(kBarOFull + ob));
      }
      __syncwarp();
      next_slot();
      ++pc;
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
