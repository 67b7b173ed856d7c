// Prefill kernel of the fully-integer attention forward for sm_100a.
//
// IntAttention (arXiv 2511.21513), "Methodology" items 2-3: int8 Q.K^T gives
// int32 scores; IndexSoftmax (row max, clipped gap, 32-entry exp LUT, int32
// sum, reciprocal multiply-shift) gives u8 probabilities; u8 x s8 P.V
// accumulates in int32 and is requantised to int8.
//
// One CTA owns one (batch, head, 128-query tile).  Warp roles:
//   warps 0-3  IndexSoftmax + epilogue; thread t owns query row t, which is
//              TMEM lane t of every accumulator (tcgen05.ld/st 32x32b).
//   warp 4     TMA producer (one thread): Q once, then K/V tiles through a
//              ring of shared-memory slots.
//   warp 5     TMEM allocator and MMA issuer (one thread): tcgen05.mma
//              kind::i8 for S = Q.K^T (both operands in shared memory) and
//              O += P.V (P from TMEM, V from shared memory, N-major).
//
// The LUT index of a score depends on the final row max and P depends on
// the final row sum Z, so a bit-exact result needs three sweeps over the
// keys of a row (online rescaling would round differently):
//   pass A  S tiles -> running row max m
//   pass B  S tiles -> Z = sum LUT[idx]; then R and the per-row table
//           Ptab[i] = (LUT[i] R + 2^31) >> 32
//   pass C  S tiles -> P = Ptab[idx] packed 4 per TMEM column -> O += P.V
// S is recomputed by the tensor cores in each pass; K streams three times
// (from L2 after the first), V once.
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
  int32_t BH, H, Lq, Lk, causal, n_qtiles, per_head;
  uint32_t lut[32];
  HeadParamsDev hp[INTATTN_MAX_HEADS];
};

namespace prefill {

constexpr int kBM = 128;       // query rows per CTA (MMA M)
constexpr int kBN = 128;       // keys per S tile (QK MMA N)
constexpr int kThreads = 192;  // 4 softmax warps + producer warp + MMA warp
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // two S buffers: [0,128) and [128,256)
constexpr uint32_t kColO = 256;  // O accumulator: d columns
constexpr uint32_t kColP = 384;  // two P buffers of 32 columns (128 u8 keys)

enum Role : unsigned { kRoleSoftmax = 1, kRoleProducer = 2, kRoleMma = 3 };

template <int D>
struct Cfg {
  static constexpr int kStages = (D == 64) ? 6 : 4;
  static constexpr uint32_t kTileBytes = kBN * D;  // one K or V tile
  static constexpr uint32_t kQBytes = kBM * D;
  static constexpr uint32_t kSwizzle = (D == 128) ? 2u : 4u;  // 128B / 64B swizzle
  static constexpr uint32_t kSBO = 8 * D;  // 8 rows of D bytes
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], s_empty[2],
  // p_full[2], p_empty[2], o_full, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 8 + 2;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kOffQ + kQBytes;
  static constexpr uint32_t kOffPtab = kOffKV + kStages * kTileBytes;
  static constexpr uint32_t kOffLut = kOffPtab + 32 * kBM * 4;
  static constexpr uint32_t kOffBars = kOffLut + 32 * 4;
  static constexpr uint32_t kOffTmem = kOffBars + kNumBars * 8;
  static constexpr uint32_t kUsed = kOffTmem + 16;
  // One CTA per SM: every CTA allocates all 512 TMEM columns, so the
  // dynamic shared memory request is padded past half of the SM's capacity.
  static constexpr uint32_t kSmemBytes = (kUsed + 1024 > 120 * 1024) ? kUsed + 1024 : 120 * 1024;
};

__device__ __forceinline__ int32_t imax(int32_t a, int32_t b) { return a > b ? a : b; }

// Requantise one int32 accumulator: clamp(floor((acc Mo + 2^(so-1)) / 2^so)).
__device__ __forceinline__ uint32_t requant_byte(int32_t acc, int32_t Mo, int32_t so) {
  const long long t = static_cast<long long>(acc) * Mo + (1ll << (so - 1));
  long long y = t >> so;  // arithmetic shift == floor division by 2^so
  y = y > 127 ? 127 : (y < -127 ? -127 : y);
  return static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(y)));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ PrefillArgs args) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sQ = s_base + C::kOffQ;
  const uint32_t sKV = s_base + C::kOffKV;
  uint32_t* ptab = reinterpret_cast<uint32_t*>(smem + C::kOffPtab);
  uint32_t* lut_s = reinterpret_cast<uint32_t*>(smem + C::kOffLut);
  const uint32_t bars = s_base + C::kOffBars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);

  const uint32_t bar_q_full = bars;
  auto bar_kv_full = [&](int i) { return bars + 8u * (1 + i); };
  auto bar_kv_empty = [&](int i) { return bars + 8u * (1 + C::kStages + i); };
  auto bar_s_full = [&](int i) { return bars + 8u * (1 + 2 * C::kStages + i); };
  auto bar_s_empty = [&](int i) { return bars + 8u * (3 + 2 * C::kStages + i); };
  auto bar_p_full = [&](int i) { return bars + 8u * (5 + 2 * C::kStages + i); };
  auto bar_p_empty = [&](int i) { return bars + 8u * (7 + 2 * C::kStages + i); };
  const uint32_t bar_o_full = bars + 8u * (9 + 2 * C::kStages);
  const uint32_t bar_drain = bars + 8u * (10 + 2 * C::kStages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- tile of this CTA (causal: the longest key ranges launch first) ----
  const int rank = blockIdx.x / args.BH;
  const int bh = blockIdx.x - rank * args.BH;
  const int qt = args.causal ? (args.n_qtiles - 1 - rank) : rank;
  const int q0 = qt * kBM;
  const int h = bh % args.H;
  const HeadParamsDev hp = args.hp[args.per_head ? h : 0];
  const int off = args.Lk - args.Lq;
  const int q_last = min(q0 + kBM, args.Lq) - 1;
  const int kend = args.causal ? min(args.Lk, q_last + off + 1) : args.Lk;
  const int nkt = (kend + kBN - 1) / kBN;

  // ---- set-up: barriers, LUT, TMEM ----
  if (tid == 0) {
    mbar_init(bar_q_full, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar_kv_full(i), 1);
      mbar_init(bar_kv_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full(i), 1);
      mbar_init(bar_s_empty(i), kBM);
      mbar_init(bar_p_full(i), kBM);
      mbar_init(bar_p_empty(i), 1);
    }
    mbar_init(bar_o_full, 1);
    mbar_init(bar_drain, 1);
    mbar_fence_init();
  }
  if (tid < 32) lut_s[tid] = args.lut[tid];
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ======================= IndexSoftmax warps =======================
    const int r = tid;  // query row within the tile == TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int row_limit = q0 + r + off;  // causal: last visible key of this row
    auto tile_full = [&](int j) {
      const int last = (j + 1) * kBN - 1;
      return last < args.Lk && (!args.causal || last <= q0 + off);
    };
    auto valid = [&](int key) { return key < args.Lk && (!args.causal || key <= row_limit); };
    bool ok = true;
    uint32_t sc = 0;  // S tiles consumed (all passes)
    auto wait_s = [&](uint32_t& buf) {
      buf = sc & 1;
      const bool got = mbar_wait(bar_s_full(buf), (sc >> 1) & 1, kRoleSoftmax);
      return __all_sync(0xffffffffu, got);
    };

    // ---- pass A: row max over valid keys ----
    int32_t m = INT_MIN;
    for (int j = 0; j < nkt; ++j, ++sc) {
      uint32_t buf;
      if (!wait_s(buf)) { ok = false; break; }
      tc_fence_after();
      const bool full = tile_full(j);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kColS + buf * kBN + c * 32, v);
        tmem_wait_ld();
        if (full) {
#pragma unroll
          for (int k = 0; k < 32; ++k) m = imax(m, static_cast<int32_t>(v[k]));
        } else {
          const int key0 = j * kBN + c * 32;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (valid(key0 + k)) m = imax(m, static_cast<int32_t>(v[k]));
        }
      }
      tc_fence_before();
      mbar_arrive(bar_s_empty(buf));
    }

    // index of a score: (min(m - S, D) M + 2^(s-1)) >> s, evaluated as
    // (C - max(S, m - D) M) >> s in wrapping 32-bit arithmetic; the true value
    // lies in [0, 2^31) so the wrap is exact.
    const long long lo64 = static_cast<long long>(m) - hp.D;
    const int32_t lo = lo64 < INT_MIN ? INT_MIN : static_cast<int32_t>(lo64);
    const uint32_t Mu = static_cast<uint32_t>(hp.M);
    const uint32_t sh = static_cast<uint32_t>(hp.s);
    const uint32_t Cm = static_cast<uint32_t>(m) * Mu + (1u << (sh - 1));

    // ---- pass B: Z = sum of pseudo-exponentials ----
    int32_t Z = 0;
    for (int j = 0; ok && j < nkt; ++j, ++sc) {
      uint32_t buf;
      if (!wait_s(buf)) { ok = false; break; }
      tc_fence_after();
      const bool full = tile_full(j);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kColS + buf * kBN + c * 32, v);
        tmem_wait_ld();
        if (full) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int32_t t = imax(static_cast<int32_t>(v[k]), lo);
            Z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(t) * Mu) >> sh]);
          }
        } else {
          // a masked key takes the clip value lo: index 31, LUT[31] = 0
          const int key0 = j * kBN + c * 32;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int32_t t = valid(key0 + k) ? imax(static_cast<int32_t>(v[k]), lo) : lo;
            Z += static_cast<int32_t>(lut_s[(Cm - static_cast<uint32_t>(t) * Mu) >> sh]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_s_empty(buf));
    }

    // reciprocal and this row's probability table
    if (ok) {
      const unsigned long long R =
          ((255ull << 32) + static_cast<unsigned long long>(Z >> 1)) / static_cast<unsigned long long>(Z);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        ptab[i * kBM + r] = static_cast<uint32_t>((static_cast<unsigned long long>(lut_s[i]) * R + (1ull << 31)) >> 32);
    }

    // ---- pass C: P tiles into TMEM for the P.V MMAs ----
    for (int j = 0; ok && j < nkt; ++j, ++sc) {
      uint32_t buf;
      if (!wait_s(buf)) { ok = false; break; }
      const uint32_t pb = j & 1;
      {
        const bool got = mbar_wait(bar_p_empty(pb), ((j >> 1) & 1) ^ 1, kRoleSoftmax);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      tc_fence_after();
      const bool full = tile_full(j);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kColS + buf * kBN + c * 32, v);
        tmem_wait_ld();
        uint32_t pw[8];
        const int key0 = j * kBN + c * 32;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint32_t word = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int k = q * 4 + b;
            // masked key: index 31, Ptab[31] = 0
            const int32_t t = (full || valid(key0 + k)) ? imax(static_cast<int32_t>(v[k]), lo) : lo;
            const uint32_t p = ptab[((Cm - static_cast<uint32_t>(t) * Mu) >> sh) * kBM + r];
            word |= p << (8 * b);
          }
          pw[q] = word;
        }
        tmem_st8(trow + kColP + pb * 32 + c * 8, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_s_empty(buf));
      mbar_arrive(bar_p_full(pb));
    }

    // ---- epilogue: O (int32, TMEM) -> requantised int8 rows ----
    if (ok) {
      const bool got = mbar_wait(bar_o_full, 0, kRoleSoftmax);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after();
      const int row = q0 + r;
      int8_t* dst = args.out + (static_cast<size_t>(bh) * args.Lq + row) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kColO + c * 32, v);
        tmem_wait_ld();
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          w[q] = requant_byte(static_cast<int32_t>(v[4 * q + 0]), hp.Mo, hp.so) |
                 (requant_byte(static_cast<int32_t>(v[4 * q + 1]), hp.Mo, hp.so) << 8) |
                 (requant_byte(static_cast<int32_t>(v[4 * q + 2]), hp.Mo, hp.so) << 16) |
                 (requant_byte(static_cast<int32_t>(v[4 * q + 3]), hp.Mo, hp.so) << 24);
        }
        if (row < args.Lq) {
          uint4* o = reinterpret_cast<uint4*>(dst + c * 32);
          o[0] = make_uint4(w[0], w[1], w[2], w[3]);
          o[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
    }
  } else if (warp == 4) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&args.tm_q);
      tma_prefetch_desc(&args.tm_k);
      tma_prefetch_desc(&args.tm_v);
      mbar_arrive_expect_tx(bar_q_full, C::kQBytes);
      tma_load_3d(sQ, &args.tm_q, bar_q_full, 0, q0, bh);
      uint32_t n = 0;  // loads issued, in the MMA warp's consumption order
      bool ok = true;
      auto load = [&](const CUtensorMap* tm, int j) {
        if (!ok) return;
        const uint32_t slot = n % C::kStages;
        const uint32_t use = n / C::kStages;
        if (!mbar_wait(bar_kv_empty(slot), (use & 1) ^ 1, kRoleProducer)) { ok = false; return; }
        mbar_arrive_expect_tx(bar_kv_full(slot), C::kTileBytes);
        tma_load_3d(sKV + slot * C::kTileBytes, tm, bar_kv_full(slot), 0, j * kBN, bh);
        ++n;
      };
      for (int pass = 0; pass < 2; ++pass)
        for (int j = 0; j < nkt; ++j) load(&args.tm_k, j);
      load(&args.tm_k, 0);
      for (int j = 0; j < nkt; ++j) {
        if (j + 1 < nkt) load(&args.tm_k, j + 1);
        load(&args.tm_v, j);
      }
      // never leave with a copy in flight: wait for the last load of each slot
      for (uint32_t slot = 0; slot < static_cast<uint32_t>(C::kStages); ++slot) {
        if (n > slot) {
          const uint32_t uses = (n - slot - 1) / C::kStages + 1;
          mbar_wait(bar_kv_full(slot), (uses - 1) & 1, kRoleProducer);
        }
      }
      mbar_wait(bar_q_full, 0, kRoleProducer);
    }
  } else {
    // ============================= MMA issuer =============================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_i8(kBM, kBN, 1, 1, 0);  // s8 x s8, K-major B
      constexpr uint32_t idesc_pv = idesc_i8(kBM, D, 0, 1, 1);    // u8 x s8, N-major B
      const uint64_t q_desc = smem_desc(sQ, 16, C::kSBO, C::kSwizzle);
      bool ok = mbar_wait(bar_q_full, 0, kRoleMma);
      uint32_t n = 0;   // K/V tiles consumed
      uint32_t sc = 0;  // S tiles produced
      auto issue_qk = [&]() {
        if (!ok) return;
        const uint32_t buf = sc & 1;
        if (!mbar_wait(bar_s_empty(buf), ((sc >> 1) & 1) ^ 1, kRoleMma)) { ok = false; return; }
        const uint32_t slot = n % C::kStages;
        if (!mbar_wait(bar_kv_full(slot), (n / C::kStages) & 1, kRoleMma)) { ok = false; return; }
        tc_fence_after();
        const uint64_t k_desc = smem_desc(sKV + slot * C::kTileBytes, 16, C::kSBO, C::kSwizzle);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)  // K = 32 bytes per MMA: advance 32 B
          mma_i8_ss(tmem + kColS + buf * kBN, q_desc + 2 * kk, k_desc + 2 * kk, idesc_qk, kk > 0);
        mma_commit(bar_kv_empty(slot));
        mma_commit(bar_s_full(buf));
        ++n;
        ++sc;
      };
      for (int t = 0; t < 2 * nkt; ++t) issue_qk();  // passes A and B
      issue_qk();                                     // pass C, tile 0
      for (int j = 0; ok && j < nkt; ++j) {
        if (j + 1 < nkt) issue_qk();
        if (!ok) break;
        const uint32_t pb = j & 1;
        if (!mbar_wait(bar_p_full(pb), (j >> 1) & 1, kRoleMma)) { ok = false; break; }
        const uint32_t slot = n % C::kStages;
        if (!mbar_wait(bar_kv_full(slot), (n / C::kStages) & 1, kRoleMma)) { ok = false; break; }
        tc_fence_after();
        const uint64_t v_desc = smem_desc(sKV + slot * C::kTileBytes, 16, C::kSBO, C::kSwizzle);
#pragma unroll
        for (int kk = 0; kk < kBN / 32; ++kk)  // 32 keys per MMA: 8 TMEM columns of P, 32 V rows
          mma_i8_ts(tmem + kColO, tmem + kColP + pb * 32 + kk * 8, v_desc + ((32u * D * kk) >> 4),
                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_kv_empty(slot));
        mma_commit(bar_p_empty(pb));
        ++n;
      }
      if (ok) mma_commit(bar_o_full);
      // every MMA this thread issued is complete before TMEM is released
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, kRoleMma);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill
}  // namespace intattn
