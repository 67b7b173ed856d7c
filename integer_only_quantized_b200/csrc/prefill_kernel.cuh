// Prefill kernel of the fully-integer attention forward for sm_100a.
//
// IntAttention (arXiv 2511.21513), "Methodology" items 2-3: int8 Q.K^T gives
// int32 scores; IndexSoftmax (row max, clipped gap, 32-entry exp LUT, int32
// sum, reciprocal multiply-shift) gives u8 probabilities; u8 x s8 P.V
// accumulates in int32 and is requantised to int8.
//
// Work unit: one (batch, head, 128-query tile).  The kernel is persistent:
// one CTA per SM takes a tile in each round, in snake order over the tiles
// sorted longest first (causal), so the loads and MMAs of a tile overlap the
// reductions of the previous one, and its epilogue the next tile's passes.
// Warp roles:
//   warps 0-15  IndexSoftmax, in two teams of eight.  Team t
//               (warps 8t .. 8t+7) takes the S tiles whose running index is
//               t mod 2, so one team computes while the other waits for its
//               next tile.  Warp w reads TMEM lane quadrant w % 4 (query rows
//               32(w%4) .. +31, one row per thread) and key half (w / 4) % 2
//               (64 of the 128 keys of an S tile).  Row max and row sum
//               combine the four partial results of a row (two teams x two
//               halves) through shared memory.
//   warp 16     TMA producer: K/V tiles through a ring of shared-memory
//               slots, one issuing lane per slot; one more lane loads Q
//               (double-buffered).
//   warp 17     TMEM allocator and MMA issuer (one thread): tcgen05.mma
//               kind::i8 for S = Q.K^T (both operands in shared memory) and
//               O += P.V (P from TMEM, V from shared memory, N-major).
//   warps 20-23 epilogue: O of a finished tile (TMEM lane quadrant
//               warp % 4, one query row per thread) -> requantised int8 rows,
//               while the softmax warps already work on the next tile.
//
// The LUT index of a score depends on the final row max and P depends on
// the final row sum Z, so a bit-exact result needs three sweeps over the
// keys of a row (online rescaling would round differently):
//   pass A  S tiles -> row max m
//   pass B  S tiles -> Z = sum LUT[idx]; then R and the per-row table
//           Ptab[i] = (LUT[i] R + 2^31) >> 32
//   pass C  S tiles -> P = Ptab[idx] packed 4 per TMEM column -> O += P.V
// S is recomputed by the tensor cores in each pass; K streams three times
// (from L2 after the first), V once.
//
// Zero-points (K and / or V as u8 codes with a zero-point per tensor or
// head): S = Q.(K - z_k) differs from Q.K_code by a per-row constant, which
// cancels in every gap m - S, so the kernel runs on the codes (the MMA reads K
// as u8).  P.(V - z_v) = P.V_code - z_v sum_j P_j: pass C also sums each
// thread's P bytes, each team then writes one correction P tile (see
// zv_correction_bytes) and the MMA warp adds it against a constant tile
// after the tile's last P.V.
//
// Every mbarrier wait is bounded (polls with a time limit).  Each softmax
// warp polls its own barriers (one vote per poll).  A warp whose wait runs
// out leaves its pass loop; every softmax warp still reaches the same
// sequence of all-warp named barriers (one per pass), which
// AND the warps' verdicts (bar.red.and), so all warps then leave together
// and none is left waiting.
#pragma once
#include <cuda.h>
#include <climits>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace intattn {

struct PrefillArgs {
  CUtensorMap tm_q;  // [B*H, Lq, d] int8, box {d, 128, 1}
  CUtensorMap tm_k;  // [B*H, Lk, d]
  CUtensorMap tm_v;  // [B*H, Lk, d]
  int8_t* out;       // [B, H, Lq, d]
  int32_t BH, H, Lq, Lk, causal, n_qtiles, per_head, n_tiles, n_luts;
  // n / BH and n / H for 0 <= n < 2^31 as (n * m) >> sh (host-computed)
  uint32_t div_bh_m, div_h_m;
  int32_t div_bh_sh, div_h_sh;
  uint32_t lut[INTATTN_MAX_CLIPS][32];  // one exp table per distinct clip threshold
  HeadParamsDev hp[INTATTN_MAX_HEADS];
  // parameters derived on the device instead (then hp is unused), and the
  // status of that derivation: the kernel writes nothing unless it is 0
  const HeadParamsDev* hp_dev;
  const uint32_t* status;
  int32_t k_u8, v_u8;  // K / V codes are u8 (they carry zero-points), else int8
};

namespace prefill {

constexpr int kBM = 128;                  // query rows per tile (MMA M)
constexpr int kBN = 128;                  // keys per S tile (QK MMA N)
#ifndef INTATTN_SOFTMAX_TEAMS
#define INTATTN_SOFTMAX_TEAMS 2
#endif
constexpr int kTeams = INTATTN_SOFTMAX_TEAMS;  // teams taking alternate S tiles
constexpr int kSoftWarps = 16;
constexpr int kTeamWarps = kSoftWarps / kTeams;
constexpr int kColGroups = kTeamWarps / 4;  // column groups per team
constexpr int kCols = kBN / kColGroups;     // S columns per thread and tile
constexpr int kGroups = kTeams * kColGroups;  // partial results per query row (= 4)
constexpr int kSoftBase = 0;               // first softmax warp
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;
// Epilogue warps 20-23 (TMEM lane quadrants 0-3); warps 18-19 only fill the
// fifth warpgroup.
constexpr int kEpiWarp0 = kSoftWarps + 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);  // 768: six whole warpgroups
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // two S buffers: [0,128) and [128,256)
constexpr uint32_t kColO = 256;  // O accumulators: d columns each (two for d = 64)
constexpr uint32_t kColP = 384;  // four P buffers of 32 columns (128 u8 keys each)
constexpr int kPBufs = 4;
// named barriers (id 0 is __syncthreads)
constexpr uint32_t kNbAll = 1;   // all softmax warps

static_assert(kGroups == 4 && kCols % 32 == 0, "4 partials per row, whole 32-column TMEM loads");

enum Role : unsigned { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3, kRoleEpilogue = 4 };

// Shared-memory barriers, by index.
enum Bar : int {
  kBarQFull = 0,        // [2]  Q tile landed
  kBarQEmpty = 2,       // [2]  every MMA reading that Q buffer is done
  kBarSFull = 4,        // [2]  S tile ready in TMEM
  kBarSEmpty = 6,       // [2]  S tile loaded by all softmax warps
  kBarPFull = 8,        // [4]  P tile written to TMEM
  kBarPEmpty = 12,      // [4]  P.V MMA that read it is done
  kBarOFull = 16,       // [2]  all P.V MMAs of a tile done (per O buffer)
  kBarOEmpty = 18,      // [2]  epilogue has read that O buffer
  kBarDrain = 20,       //      final MMA drain
  kBarKvFull = 21,      // [stages], then kv_empty[stages]
};

// ZV: the kernel instance that supports a V zero-point (the correction tile
// and the sums of P); the other instance is the plain int8 kernel.
template <int D, bool ZV = false>
struct Cfg {
  static constexpr int kStages = (D == 64) ? 8 : 6;
  // O accumulators in TMEM: with d = 64 two fit below the P buffers, so a
  // tile accumulates into one while the epilogue drains the other
  static constexpr int kOBufs = (D == 64) ? 2 : 1;
  static_assert(kColO + kOBufs * D <= kColP, "O buffers overlap the P buffers");
  static constexpr uint32_t kTileBytes = kBN * D;  // one K or V tile
  static constexpr uint32_t kQBytes = kBM * D;
  static constexpr uint32_t kSwizzle = (D == 128) ? 2u : 4u;  // 128B / 64B swizzle
  static constexpr uint32_t kSBO = 8 * D;  // 8 rows of D bytes
  static constexpr int kNumBars = kBarKvFull + 2 * kStages;
  static constexpr uint32_t kOffQ = 0;                                  // [2] Q tiles
  static constexpr uint32_t kOffKV = kOffQ + 2 * kQBytes;
  // constant s8 tile [32 keys][D] of the V zero-point correction (rows 16 g:
  // -1, rows 16 g + 1 .. 16 g + 4: -128, else 0), laid out like a V tile
  static constexpr uint32_t kOffCorr = kOffKV + kStages * kTileBytes;
  static constexpr int kCorrGroup = 16;  // keys of a correction tile per partial owner (two per team)
  // probability table, four copies [b][33][kBM] u32 with P << 8b, so four
  // looked-up bytes pack into a word by integer adds
  static constexpr uint32_t kPtabBytes = 33 * kBM * 4;
  static constexpr uint32_t kOffPtab = kOffCorr + (ZV ? 32 * D : 0);
  static constexpr uint32_t kOffRed = kOffPtab + 4 * kPtabBytes;        // [2][kGroups][kBM] int32
  static constexpr uint32_t kOffLut = kOffRed + 2 * kGroups * kBM * 4;
  static constexpr uint32_t kOffHp = kOffLut + INTATTN_MAX_CLIPS * 32 * 4;  // head parameters
  static constexpr uint32_t kOffBars = kOffHp + INTATTN_MAX_HEADS * sizeof(HeadParamsDev);
  static constexpr uint32_t kOffTmem = kOffBars + kNumBars * 8;
  static constexpr uint32_t kUsed = kOffTmem + 16;
  // One CTA per SM: every CTA allocates all 512 TMEM columns, so the
  // dynamic shared memory request is padded past half of the SM's capacity.
  static constexpr uint32_t kSmemBytes = (kUsed + 1024 > 120 * 1024) ? kUsed + 1024 : 120 * 1024;
};

__device__ __forceinline__ int32_t imax(int32_t a, int32_t b) { return a > b ? a : b; }

// a b + c, rounded toward zero, then clamped to [0, 1] (one fma.rz.sat).
__device__ __forceinline__ float fma_rz_sat(float a, float b, float c) {
  float d;
  asm("fma.rz.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (a0, a1) * b + c in both lanes, rounded toward zero: one packed FP32 FMA.
// b2 and c2 hold the multiplier and addend twice (pack2 below).
__device__ __forceinline__ void fma2_rz(float a0, float a1, unsigned long long b2, unsigned long long c2,
                                        float& d0, float& d1) {
  asm("{\n\t.reg .b64 a, d;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "fma.rz.f32x2 d, a, %4, %5;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "l"(b2), "l"(c2));
}

__device__ __forceinline__ unsigned long long pack2(float x) {
  const unsigned long long u = __float_as_uint(x);
  return u | (u << 32);
}

// R = floor((255 2^32 + floor(Z/2)) / Z), Z >= 1: N < 2^40, so the double
// quotient is within one unit of R, and one integer step makes it exact.
__device__ __forceinline__ unsigned long long exact_R(int32_t Z) {
  const unsigned long long N = (255ull << 32) + static_cast<unsigned long long>(Z >> 1);
  const unsigned long long Zu = static_cast<unsigned long long>(Z);
  unsigned long long R = static_cast<unsigned long long>(__ddiv_rn(static_cast<double>(N), static_cast<double>(Z)));
  if (R * Zu > N) --R;
  else if ((R + 1) * Zu <= N) ++R;
  return R;
}

// Requantise one int32 accumulator: clamp(floor((acc Mo + 2^(so-1)) / 2^so)).
__device__ __forceinline__ uint32_t requant_byte(int32_t acc, int32_t Mo, int32_t so) {
  const long long t = static_cast<long long>(acc) * Mo + (1ll << (so - 1));
  long long y = t >> so;  // arithmetic shift == floor division by 2^so
  y = y > 127 ? 127 : (y < -127 ? -127 : y);
  return static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(y)));
}

// Four u8 values (each < 256 in a 32-bit register) into one word, byte k = p_k.
__device__ __forceinline__ uint32_t pack4(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3) {
  return __byte_perm(__byte_perm(p0, p1, 0x3340), __byte_perm(p2, p3, 0x3340), 0x5410);
}

// Geometry of one work unit.
struct Tile {
  int bh, h, q0, nkt;
};

// Tile of round `round` for CTA `cta`: rounds alternate direction over the
// tiles (sorted longest first for causal), which evens out the work per CTA.
__device__ __forceinline__ int tile_index(int round, int cta, int ctas) {
  return round * ctas + ((round & 1) ? (ctas - 1 - cta) : cta);
}

// floor(n / d) for 0 <= n < 2^31 with the multiplier and shift of d.
__device__ __forceinline__ int fast_div(int n, uint32_t m, int sh) {
  return static_cast<int>((static_cast<unsigned long long>(static_cast<uint32_t>(n)) * m) >> sh);
}

__device__ __forceinline__ Tile tile_of(const PrefillArgs& a, int L) {
  Tile t;
  const int rank = fast_div(L, a.div_bh_m, a.div_bh_sh);
  t.bh = L - rank * a.BH;
  const int qt = a.causal ? (a.n_qtiles - 1 - rank) : rank;
  t.q0 = qt * kBM;
  t.h = t.bh - fast_div(t.bh, a.div_h_m, a.div_h_sh) * a.H;
  const int off = a.Lk - a.Lq;
  const int q_last = min(t.q0 + kBM, a.Lq) - 1;
  const int kend = a.causal ? min(a.Lk, q_last + off + 1) : a.Lk;
  t.nkt = (kend + kBN - 1) / kBN;
  return t;
}

template <int D, bool ZV>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ PrefillArgs args) {
  using C = Cfg<D, ZV>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (swizzled TMA tiles); offsetting the __shared__
  // array keeps the compiler aware of the address space.
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

  // ---- set-up: barriers, LUT, TMEM (once per CTA) ----
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarQFull + i), 1);
      mbar_init(bar(kBarQEmpty + i), 1);
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), kTeamWarps);
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(bar(kBarPFull + i), kTeamWarps);
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
    // the zero-point correction tile (uniform rows: the swizzle moves bytes within a row only)
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

  if (warp >= kSoftBase && warp < kSoftBase + kSoftWarps) {
    // ======================= IndexSoftmax warps =======================
    // A warp reaches the TMEM lanes of quadrant warp % 4; four consecutive
    // softmax warps cover the four quadrants.
    const int sw = warp - kSoftBase;
    const int quad = warp & 3;
    const int half = (sw >> 2) % kColGroups;  // column group within the team
    const int team = sw / kTeamWarps;
    const int grp = team * kColGroups + half;   // slot of this thread's partial results
    const int r = quad * 32 + lane;   // query row within the tile == TMEM lane
    const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t trow = tlane + half * kCols;
    const uint32_t prow = smem_u32(ptab) + 4u * r;  // row k of the table at prow + 512 k
    // The index code k of a score (see idx_bits below) is idx + 1, or 0 / 32
    // for a masked / clipped key.  Lane k holds LUT[k-1] as a float (lane 0:
    // 0); a shuffle whose source lane is the low 5 bits of the code looks it
    // up.  Per tile a thread sums 32 values below 2^15: the float sums are exact.
    int32_t lut_lane = 0;  // set per tile: the table of the tile's head
    if (sw < 4)
      for (int b = 0; b < 4; ++b) ptab[b * (C::kPtabBytes / 4) + r] = 0u;  // table row 0 (masked keys) stays 0
    bool ok = true;
    uint32_t sc = 0;  // S tiles of the CTA so far (both teams, all passes and tiles)
    uint32_t pc = 0;  // P tiles of the CTA so far
    // wait for a barrier phase (every warp polls for itself: a leader that
    // polls and wakes its team through a named barrier adds that barrier's
    // latency to every S tile)
    auto team_wait = [&](uint32_t b, uint32_t parity) { return mbar_wait_warp(b, parity, kRoleSoftmax); };
    // all sixteen softmax warps: every warp's `ok`, and (softmax warp 0 polling) a phase
    auto all_sync = [&](bool mine) { return bar_red_and(kNbAll, 32 * kSoftWarps, mine); };
    auto arrive_warp = [&](uint32_t b) {  // one arrival per warp
      __syncwarp();
      if (lane == 0) mbar_arrive(b);
    };
    // S tile `idx` in 32-column chunks: load chunk c, then body(v, c); the
    // buffer is released after its last chunk is loaded, so only 32 scores
    // per thread are live at a time.
    auto walk_s = [&](uint32_t idx, auto&& body) {
      const uint32_t buf = idx & 1;
      if (!team_wait(bar(kBarSFull + buf), (idx >> 1) & 1)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kCols / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kColS + buf * kBN + 32 * c, v);
        tmem_wait_ld();
        if (c == kCols / 32 - 1) {
          tc_fence_before();
          arrive_warp(bar(kBarSEmpty + buf));
        }
        body(v, c);
      }
      return true;
    };
    // first tile of a pass of nkt tiles that belongs to this team
    auto first_j = [&](uint32_t s0) {
      return kTeams == 1 ? 0 : static_cast<int>((static_cast<uint32_t>(team) - s0) & 1u);
    };

    for (int it = 0; ok; ++it) {
      const int L = tile_index(it, blockIdx.x, gridDim.x);
      if (L >= args.n_tiles) break;
      const Tile T = tile_of(args, L);
      const HeadParamsDev hp = hp_s[args.per_head ? T.h : 0];
      const uint32_t* lut_h = lut_s + 32 * hp.lut;
      lut_lane = __float_as_int(lane == 0 ? 0.f : __int2float_rn(static_cast<int32_t>(lut_h[lane - 1])));
      const int off = args.Lk - args.Lq;
      const int row_limit = T.q0 + r + off;  // causal: last visible key of this row
      auto tile_full = [&](int j) {
        const int last = (j + 1) * kBN - 1;
        return last < args.Lk && (!args.causal || last <= T.q0 + off);
      };
      // keys of this thread's segment of tile j that are visible: a prefix
      const int key_lim = args.causal ? min(args.Lk, row_limit + 1) : args.Lk;
      auto nvalid = [&](int j) { return min(max(key_lim - (j * kBN + half * kCols), 0), kCols); };

      // ---- pass A: row max over valid keys ----
      int32_t m = INT_MIN;
      for (int j = first_j(sc); j < T.nkt; j += kTeams) {
        int32_t m4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
        const bool full = tile_full(j);
        const int nv = nvalid(j);
        const bool got = walk_s(sc + j, [&](const uint32_t (&v)[32], int c) {
          if (full) {
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
              m4[0] = __vimax3_s32(m4[0], static_cast<int32_t>(v[k + 0]), static_cast<int32_t>(v[k + 1]));
              m4[1] = __vimax3_s32(m4[1], static_cast<int32_t>(v[k + 2]), static_cast<int32_t>(v[k + 3]));
              m4[2] = __vimax3_s32(m4[2], static_cast<int32_t>(v[k + 4]), static_cast<int32_t>(v[k + 5]));
              m4[3] = __vimax3_s32(m4[3], static_cast<int32_t>(v[k + 6]), static_cast<int32_t>(v[k + 7]));
            }
          } else {
            const int nc = nv - 32 * c;
#pragma unroll
            for (int k = 0; k < 32; ++k)
              m4[k & 3] = imax(m4[k & 3], k < nc ? static_cast<int32_t>(v[k]) : INT_MIN);
          }
        });
        if (!got) { ok = false; break; }
        m = imax(m, imax(imax(m4[0], m4[1]), imax(m4[2], m4[3])));
      }
      sc += T.nkt;
      red[grp * kBM + r] = m;
      if (!all_sync(ok)) { ok = false; break; }
      m = imax(imax(red[r], red[kBM + r]), imax(red[2 * kBM + r], red[3 * kBM + r]));

      // LUT index of a score, idx = floor((min(m - S, D) M + 2^(s-1)) / 2^s),
      // evaluated exactly on the FP32 pipe (the integer pipe is the scarcer
      // one), as the code k = idx + 1 (idx <= 30) or k = 32 (clipped):
      //  * (0x4B000000 + m) - S, read as a float, is X = 2^23 + g exactly,
      //    g = m - S in [0, 2^22];
      //  * with v = g M / 2^s + 1/2, the definition's index is min(floor(v), 31):
      //    D is the smallest gap whose index reaches 31 and M <= 2^s;
      //  * every valid parameter set has s in {24, 25, 26}, so Ms' = M 2^-(s+5)
      //    and c1 = (3/2 - 2^23 M 2^-s) / 32 are exact floats, and
      //    X Ms' + c1 = (v + 1) / 32; one fma rounded toward zero and saturated
      //    to [0, 1] gives y = min(RZ((v + 1) / 32), 1);
      //  * 32 y + 2^23 rounded toward zero is 2^23 + min(floor(v) + 1, 32) (the
      //    scaling by 32 commutes with the rounding), so the bits are
      //    0x4B000000 + k: the low 5 bits are k mod 32, and (bits * 512) mod
      //    2^32 is k * 512, the offset of row k of the table.
      // A masked key uses the bits 0x4B000000: code 0, lane 0 and row 0 hold 0.
      const uint32_t Cx = 0x4B000000u + static_cast<uint32_t>(m);
      const float Mf = __int2float_rn(hp.M);                                                   // exact: M <= 2^24
      const float Ms32 = Mf * __uint_as_float(static_cast<uint32_t>(127 - 5 - hp.s) << 23);   // M 2^-(s+5)
      const float c1 = (1.5f - Mf * __uint_as_float(static_cast<uint32_t>(127 + 23 - hp.s) << 23)) * 0.03125f;
      auto idx_bits = [&](uint32_t sv) {
        const float y = fma_rz_sat(__uint_as_float(Cx - sv), Ms32, c1);
        return __float_as_uint(__fmaf_rz(y, 32.0f, 8388608.0f));
      };
      // the same for two scores, the second multiply-add as one packed instruction
      auto idx_bits2 = [&](uint32_t s0, uint32_t s1, uint32_t& b0, uint32_t& b1) {
        const float y0 = fma_rz_sat(__uint_as_float(Cx - s0), Ms32, c1);
        const float y1 = fma_rz_sat(__uint_as_float(Cx - s1), Ms32, c1);
        float k0, k1;
        fma2_rz(y0, y1, pack2(32.0f), pack2(8388608.0f), k0, k1);
        b0 = __float_as_uint(k0);
        b1 = __float_as_uint(k1);
      };
      constexpr uint32_t kMaskedBits = 0x4B000000u;

      // ---- pass B: Z = sum of pseudo-exponentials ----
      int32_t Z = 0;
      for (int j = first_j(sc); j < T.nkt; j += kTeams) {
        float z4[4] = {0.f, 0.f, 0.f, 0.f};
        const bool full = tile_full(j);
        const int nv = nvalid(j);
        const bool got = walk_s(sc + j, [&](const uint32_t (&v)[32], int c) {
          if (full) {
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              uint32_t b0, b1;
              idx_bits2(v[k], v[k + 1], b0, b1);
              z4[k & 3] += __int_as_float(__shfl_sync(0xffffffffu, lut_lane, static_cast<int>(b0)));
              z4[(k + 1) & 3] += __int_as_float(__shfl_sync(0xffffffffu, lut_lane, static_cast<int>(b1)));
            }
          } else {
            const int nc = nv - 32 * c;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const uint32_t ib = k < nc ? idx_bits(v[k]) : kMaskedBits;
              z4[k & 3] += __int_as_float(__shfl_sync(0xffffffffu, lut_lane, static_cast<int>(ib)));
            }
          }
        });
        if (!got) { ok = false; break; }
        Z += __float2int_rn((z4[0] + z4[1]) + (z4[2] + z4[3]));
      }
      sc += T.nkt;
      red[(kGroups + grp) * kBM + r] = Z;
      if (!all_sync(ok)) { ok = false; break; }
      Z = (red[kGroups * kBM + r] + red[(kGroups + 1) * kBM + r]) +
          (red[(kGroups + 2) * kBM + r] + red[(kGroups + 3) * kBM + r]);

      // reciprocal and this row's probability table: row k = Ptab[k - 1]
      // (each of the four threads of a row writes 8 of the rows 1..32)
      {
        const unsigned long long R = exact_R(Z);
#pragma unroll
        for (int i = grp * 8; i < grp * 8 + 8; ++i) {
          const uint32_t P = static_cast<uint32_t>((static_cast<unsigned long long>(lut_h[i]) * R + (1ull << 31)) >> 32);
#pragma unroll
          for (int b = 0; b < 4; ++b) ptab[b * (C::kPtabBytes / 4) + (i + 1) * kBM + r] = P << (8 * b);
        }
      }
      all_sync(true);  // the table is complete

      // ---- pass C: P tiles into TMEM for the P.V MMAs ----
      const bool corr = ZV && hp.zv != 0;  // V zero-point: sum this thread's P bytes
      uint32_t psum = 0;
      for (int j = first_j(sc); j < T.nkt; j += kTeams) {
        const uint32_t pi = pc + j;  // running P index of this tile
        const uint32_t pb = pi & (kPBufs - 1);
        if (!team_wait(bar(kBarPEmpty + pb), ((pi / kPBufs) & 1) ^ 1)) { ok = false; break; }
        const bool full = tile_full(j);
        const int nv = nvalid(j);
        const bool got = walk_s(sc + j, [&](const uint32_t (&v)[32], int c) {
          uint32_t pw[8];
          if (full) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              uint32_t kb[4], p[4];
              idx_bits2(v[q * 4], v[q * 4 + 1], kb[0], kb[1]);
              idx_bits2(v[q * 4 + 2], v[q * 4 + 3], kb[2], kb[3]);
#pragma unroll
              for (int b = 0; b < 4; ++b) p[b] = lds_u32(kb[b] * 512u + prow + b * C::kPtabBytes);
              pw[q] = (p[0] + p[1]) + (p[2] + p[3]);
            }
          } else {
            const int nc = nv - 32 * c;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              uint32_t p[4];
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const int k = q * 4 + b;
                const uint32_t ib = k < nc ? idx_bits(v[k]) : kMaskedBits;
                p[b] = lds_u32(ib * 512u + prow + b * C::kPtabBytes);
              }
              pw[q] = (p[0] + p[1]) + (p[2] + p[3]);
            }
          }
          if (corr) {
#pragma unroll
            for (int q = 0; q < 8; ++q) psum = __dp4a(pw[q], 0x01010101u, psum);
          }
          tmem_st8(tlane + kColP + pb * 32 + half * (kCols / 4) + c * 8, pw);
        });
        if (!got) { ok = false; break; }
        tmem_wait_st();
        tc_fence_before();
        arrive_warp(bar(kBarPFull + pb));
      }
      if (corr && ok) {
        // this team's correction tile: P index pc + nkt + team, keys
        // kCorrGroup * half .. of it hold this thread's share
        const uint32_t pi = pc + T.nkt + team;
        const uint32_t pb = pi & (kPBufs - 1);
        if (!team_wait(bar(kBarPEmpty + pb), ((pi / kPBufs) & 1) ^ 1)) {
          ok = false;
        } else {
          uint32_t w0, w1;
          zv_correction_bytes(hp.zv * static_cast<int32_t>(psum), w0, w1);
          tmem_st4(tlane + kColP + pb * 32 + half * (C::kCorrGroup / 4), w0, w1, 0u, 0u);
          tmem_wait_st();
          tc_fence_before();
          arrive_warp(bar(kBarPFull + pb));
        }
      }
      sc += T.nkt;
      pc += T.nkt + (corr ? kTeams : 0);

    }
  } else if (warp >= kEpiWarp0) {
    // ============================ epilogue ============================
    // O (int32, TMEM) of each tile -> requantised int8 rows, while the
    // softmax warps go on with the next tile.  Thread = query row (TMEM lane).
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
        if (c == D / 16 - 1) {  // O may now be overwritten by the next tile
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
    // The tensor loads one thread issues are served one after another, so a
    // single issuing thread caps the load rate of the SM far below what the
    // passes consume.  Lane s < kStages therefore owns ring slot s and issues
    // every K/V load that lands there (load n goes to slot n % kStages), and
    // lane kQLane issues the Q loads.  Each lane walks the same load sequence
    // and waits, with the per-thread bounded wait, only on its own barriers.
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
      uint32_t n = 0;     // position in the K/V load sequence (MMA consumption order)
      uint32_t mine = 0;  // loads this lane issued
      bool ok = true;
      auto load = [&](const CUtensorMap* tm, int j, int bh) {
        if (ok && n % C::kStages == slot) {
          if (!mbar_wait(bar_kv_empty(slot), (mine & 1) ^ 1, kRoleProducer)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(bar_kv_full(slot), C::kTileBytes);
            tma_load_3d(dst, tm, bar_kv_full(slot), 0, j * kBN, bh);
            ++mine;
          }
        }
        ++n;
      };
      for (int it = 0; ok; ++it) {
        const int L = tile_index(it, blockIdx.x, gridDim.x);
        if (L >= args.n_tiles) break;
        const Tile T = tile_of(args, L);
        for (int pass = 0; pass < 2; ++pass)
          for (int j = 0; j < T.nkt; ++j) load(&args.tm_k, j, T.bh);
        load(&args.tm_k, 0, T.bh);
        if (T.nkt > 1) load(&args.tm_k, 1, T.bh);
        for (int j = 0; j < T.nkt; ++j) {
          if (j + 2 < T.nkt) load(&args.tm_k, j + 2, T.bh);
          load(&args.tm_v, j, T.bh);
        }
      }
      // never leave with a copy in flight: wait for this slot's last load
      if (mine > 0) mbar_wait(bar_kv_full(slot), (mine - 1) & 1, kRoleProducer);
    } else if (lane == kQLane) {
      uint32_t nq = 0;  // Q loads issued
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
        const uint32_t last = nq - 1 - i;  // the last load of each Q buffer
        mbar_wait(bar(kBarQFull + (last & 1)), (last >> 1) & 1, kRoleProducer);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ============================= MMA issuer =============================
    // The whole warp runs this loop on uniform values (descriptors stay in
    // uniform registers) and waits for both inputs of an MMA group with one
    // vote per poll; one elected lane issues the group and its commits.
    const uint32_t idesc_qk = idesc_i8(kBM, kBN, 1, args.k_u8 ? 0u : 1u, 0);  // s8 x (s8 | u8), K-major B
    const uint32_t idesc_pv = idesc_i8(kBM, D, 0, args.v_u8 ? 0u : 1u, 1);    // u8 x (s8 | u8), N-major B
    constexpr uint32_t idesc_corr = idesc_i8(kBM, D, 0, 1, 1);                // u8 x s8: the correction tile
    const uint64_t kv_desc0 = smem_desc(sKV, 16, C::kSBO, C::kSwizzle);
    const uint64_t corr_desc = smem_desc(s_base + C::kOffCorr, 16, C::kSBO, C::kSwizzle);
    constexpr uint32_t kSlotDesc = C::kTileBytes >> 4;  // descriptor step between ring slots
    bool ok = true;
    uint32_t slot = 0, kv_par = 0;  // ring slot and phase parity of the next K/V tile
    uint32_t sc = 0;  // S tiles produced
    uint32_t pc = 0;  // P tiles consumed
    auto next_slot = [&]() {
      if (++slot == static_cast<uint32_t>(C::kStages)) {
        slot = 0;
        kv_par ^= 1;
      }
    };
    for (int it = 0; ok; ++it) {
      const int L = tile_index(it, blockIdx.x, gridDim.x);
      if (L >= args.n_tiles) break;
      const Tile T = tile_of(args, L);
      const uint32_t qb = it & 1;
      if (!mbar_wait_warp(bar(kBarQFull + qb), (it >> 1) & 1, kRoleMma)) { ok = false; break; }
      const uint64_t q_desc = smem_desc(sQ(qb), 16, C::kSBO, C::kSwizzle);
      auto issue_qk = [&]() {
        if (!ok) return;
        const uint32_t buf = sc & 1;
        if (!mbar_wait2_warp(bar(kBarSEmpty + buf), ((sc >> 1) & 1) ^ 1, bar_kv_full(slot), kv_par, kRoleMma)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint64_t k_desc = kv_desc0 + slot * kSlotDesc;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)  // K = 32 bytes per MMA: advance 32 B
            mma_i8_ss(tmem + kColS + buf * kBN, q_desc + 2 * kk, k_desc + 2 * kk, idesc_qk, kk > 0);
          mma_commit(bar_kv_empty(slot));
          mma_commit(bar(kBarSFull + buf));
        }
        __syncwarp();
        next_slot();
        ++sc;
      };
      for (int t = 0; t < 2 * T.nkt; ++t) issue_qk();  // passes A and B
      // pass C: S tile j+2 reuses the buffer of tile j, which the softmax
      // warps release right after loading it, so QK(j+2) goes before P.V(j)
      issue_qk();
      if (T.nkt > 1) issue_qk();
      for (int j = 0; ok && j < T.nkt; ++j, ++pc) {
        if (j + 2 < T.nkt) issue_qk();
        if (!ok) break;
        // O of the previous tile must have been read before it is overwritten
        // (with two O buffers: the tile before the previous one)
        if (j == 0 && !mbar_wait_warp(bar(kBarOEmpty + it % C::kOBufs), ((it / C::kOBufs) & 1) ^ 1, kRoleMma)) {
          ok = false;
          break;
        }
        const uint32_t pb = pc & (kPBufs - 1);
        if (!mbar_wait2_warp(bar(kBarPFull + pb), (pc / kPBufs) & 1, bar_kv_full(slot), kv_par, kRoleMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t v_desc = kv_desc0 + slot * kSlotDesc;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk)  // 32 keys per MMA: 8 TMEM columns of P, 32 V rows
            mma_i8_ts(tmem + kColO + (it % C::kOBufs) * D, tmem + kColP + pb * 32 + kk * 8,
                      v_desc + ((32u * D * kk) >> 4), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_kv_empty(slot));
          mma_commit(bar(kBarPEmpty + pb));
        }
        __syncwarp();
        next_slot();
      }
      if (!ok) break;
      if (ZV && hp_s[args.per_head ? T.h : 0].zv != 0) {
        // O -= z_v sum_j P_j: one correction tile per softmax team
        for (int t = 0; t < kTeams; ++t, ++pc) {
          const uint32_t pb = pc & (kPBufs - 1);
          if (!mbar_wait_warp(bar(kBarPFull + pb), (pc / kPBufs) & 1, kRoleMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            mma_i8_ts(tmem + kColO + (it % C::kOBufs) * D, tmem + kColP + pb * 32, corr_desc, idesc_corr, 1u);
            mma_commit(bar(kBarPEmpty + pb));
          }
          __syncwarp();
        }
        if (!ok) break;
      }
      mma_commit_elect(bar(kBarQEmpty + qb));  // every MMA that read this Q buffer
      mma_commit_elect(bar(kBarOFull + it % C::kOBufs));
    }
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

}  // namespace prefill
}  // namespace intattn
