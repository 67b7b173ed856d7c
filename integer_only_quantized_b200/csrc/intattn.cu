// C ABI of the fully-integer attention forward (see include/intattn.h).
//
// Host side: argument checks, the integer parameters of every head (IEEE
// double, the order of operations fixed by the definition in intattn.h),
// TMA descriptors, and launches on the caller's stream.  Device side: the
// kernels in prefill_kernel.cuh and decode_kernel.cuh, compiled into this
// single translation unit for sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "intattn.h"

#include "calibrate_kernel.cuh"
#include "decode_kernel.cuh"
#include "gelu_kernel.cuh"
#include "params_kernel.cuh"
#include "quantize_kernel.cuh"
#include "prefill_kernel.cuh"
#include "prefill_short_kernel.cuh"

using intattn::DecodeArgs;
using intattn::HeadParamsDev;
using intattn::PrefillArgs;

namespace {

// ----------------------------------------------------------------- params
// Index multiplier/shift/clip of one head: M / 2^s approximates
// alpha * 31 / c with alpha = s_q s_k / sqrt(d); D is the first gap whose
// rounded index is 31.
int index_params(double s_q, double s_k, int d, double c, HeadParamsDev* hp) {
  if (!std::isfinite(s_q) || !std::isfinite(s_k) || !std::isfinite(c)) return INTATTN_ERR_PARAM_RANGE;
  if (!(s_q > 0.0) || !(s_k > 0.0) || !(c > 0.0)) return INTATTN_ERR_PARAM_RANGE;
  const double alpha = (s_q * s_k) / std::sqrt(static_cast<double>(d));
  const double steps_per_unit = (alpha * 31.0) / c;
  int shift = 26;
  long long mult = std::llround(std::ldexp(steps_per_unit, shift));
  while (shift > 1 && mult > (1ll << 24)) {
    --shift;
    mult = std::llround(std::ldexp(steps_per_unit, shift));
  }
  if (mult < 1 || mult > (1ll << 24) || mult > (1ll << shift)) return INTATTN_ERR_PARAM_RANGE;
  const long long half_steps = 61ll << (shift - 1);  // 30.5 index steps, in units of 2^-s
  hp->M = static_cast<int32_t>(mult);
  hp->s = shift;
  hp->D = static_cast<int32_t>((half_steps + mult - 1) / mult);
  return INTATTN_OK;
}

// Requantisation multiplier/shift: acc * s_v / (255 s_o) ~= acc * Mo / 2^so.
int requant_params(double s_v, double s_o, HeadParamsDev* hp) {
  if (!std::isfinite(s_v) || !std::isfinite(s_o) || !(s_v > 0.0) || !(s_o > 0.0))
    return INTATTN_ERR_PARAM_RANGE;
  int e = 0;
  const double f = std::frexp(s_v / (255.0 * s_o), &e);  // f in [0.5, 1)
  long long mo = std::llround(f * 2147483648.0);
  if (mo == (1ll << 31)) {
    mo = 1ll << 30;
    ++e;
  }
  const int so = 31 - e;
  if (so < 1 || so > 62) return INTATTN_ERR_PARAM_RANGE;
  hp->Mo = static_cast<int32_t>(mo);
  hp->so = so;
  return INTATTN_OK;
}

int make_lut(double c, uint32_t lut[32]) {
  if (!std::isfinite(c) || !(c > 0.0)) return INTATTN_ERR_PARAM_RANGE;
  for (int i = 0; i < 31; ++i)
    lut[i] = static_cast<uint32_t>(std::llround(32768.0 * std::exp(-(static_cast<double>(i) * c) / 31.0)));
  lut[31] = 0u;  // a clipped gap contributes nothing
  return INTATTN_OK;
}

// LUTs and head parameters; per-tensor scales fill hp[0] only.  Each
// distinct clip threshold gets its own table (at most INTATTN_MAX_CLIPS).
int derive(const intattn_scales_t* sc, int H, int d, float clip_c, uint32_t lut[INTATTN_MAX_CLIPS][32],
           HeadParamsDev* hp, int max_heads, int* n_luts = nullptr) {
  if (!sc || !sc->s_q || !sc->s_k || !sc->s_v || !sc->s_o) return INTATTN_ERR_INVALID_ARG;
  if (H <= 0) return INTATTN_ERR_INVALID_ARG;
  const int n = sc->per_head ? H : 1;
  if (n > max_heads) return INTATTN_ERR_UNSUPPORTED;
  float clips[INTATTN_MAX_CLIPS];
  int nclips = 0;
  for (int i = 0; i < n; ++i) {
    const float c = sc->clip_c ? sc->clip_c[i] : clip_c;
    int id = 0;
    while (id < nclips && !(clips[id] == c)) ++id;
    if (id == nclips) {
      if (nclips == INTATTN_MAX_CLIPS) return INTATTN_ERR_UNSUPPORTED;
      const int rc = make_lut(static_cast<double>(c), lut[nclips]);
      if (rc) return rc;
      clips[nclips++] = c;
    }
    int rc = index_params(sc->s_q[i], sc->s_k[i], d, static_cast<double>(c), &hp[i]);
    if (rc) return rc;
    rc = requant_params(sc->s_v[i], sc->s_o[i], &hp[i]);
    if (rc) return rc;
    hp[i].lut = id;
    // zero-points: u8 codes, 0 .. 255 (K's cancels in every gap: checked only)
    if (sc->z_k && (sc->z_k[i] < 0 || sc->z_k[i] > 255)) return INTATTN_ERR_INVALID_ARG;
    if (sc->z_v && (sc->z_v[i] < 0 || sc->z_v[i] > 255)) return INTATTN_ERR_INVALID_ARG;
    hp[i].zv = sc->z_v ? sc->z_v[i] : 0;
  }
  if (n_luts) *n_luts = nclips;
  return INTATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Multiplier and shift with floor(n / d) == (n m) >> sh for every 0 <= n < 2^31
// and d >= 1: m = ceil(2^(31 + l) / d), sh = 31 + l, l = ceil(log2 d) (the
// round-up reciprocal of Granlund and Montgomery for 31-bit dividends; m < 2^32).
void div_magic(uint32_t d, uint32_t* m, int32_t* sh) {
  int l = 0;
  while ((1ull << l) < d) ++l;
  const int k = 31 + l;
  *m = static_cast<uint32_t>(((1ull << k) + d - 1) / d);
  *sh = k;
}

// ------------------------------------------------------------------- TMA
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [planes, rows, d] int8 tensor, box {d, box_rows, 1}, swizzle = d bytes.
bool encode_3d(CUtensorMap* m, const void* base, int d, long long rows, long long planes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows) * d};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(d), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle sw = (d == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Multiprocessor count of the current device (cached per device).
int sm_count(int* out) {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return INTATTN_ERR_CUDA;
    cache[dev] = v;
  }
  *out = cache[dev];
  return INTATTN_OK;
}

// Text of the last CUDA error a launch reported (this thread), for
// intattn_strerror(INTATTN_ERR_CUDA).
thread_local const char* g_last_cuda_error = nullptr;

int note_launch(cudaError_t e) {
  if (e == cudaSuccess) return INTATTN_OK;
  g_last_cuda_error = cudaGetErrorString(e);
  return INTATTN_ERR_CUDA;
}

// ------------------------------------------------------- kernel attributes
template <int D, bool ZV>
int prefill_launch(const PrefillArgs& args, int grid, cudaStream_t stream) {
  using C = intattn::prefill::Cfg<D, ZV>;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return INTATTN_ERR_CUDA;
  if (dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(intattn::prefill::prefill_kernel<D, ZV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmemBytes)) != cudaSuccess)
      return INTATTN_ERR_CUDA;
    attr_set[dev] = true;
  }
  intattn::prefill::prefill_kernel<D, ZV><<<grid, intattn::prefill::kThreads, C::kSmemBytes, stream>>>(args);
  return note_launch(cudaGetLastError());
}

template <int D, bool ZV>
int prefill_short_launch(const PrefillArgs& args, int grid, cudaStream_t stream) {
  using C = intattn::shortrow::Cfg<D, ZV>;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return INTATTN_ERR_CUDA;
  if (dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(intattn::shortrow::prefill_short_kernel<D, ZV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmemBytes)) != cudaSuccess)
      return INTATTN_ERR_CUDA;
    attr_set[dev] = true;
  }
  intattn::shortrow::prefill_short_kernel<D, ZV><<<grid, intattn::shortrow::kThreads, C::kSmemBytes, stream>>>(args);
  return note_launch(cudaGetLastError());
}

struct DecodeLayout {
  int nsplit, ld_s;
  size_t off_s, off_max, off_part, off_cnt, off_mr, total;
};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// chunk: keys per CTA of the split; the int8 value gives the largest layout
DecodeLayout decode_layout(long long BH, int Lk, int d, int chunk = intattn::decode::kChunk) {
  DecodeLayout L{};
  L.nsplit = (Lk + chunk - 1) / chunk;
  L.off_s = 0;
  L.ld_s = (Lk + 3) & ~3;  // 16-byte aligned score rows
  L.off_max = L.off_s + round256(static_cast<size_t>(BH) * L.ld_s * 4);
  L.off_part = L.off_max + round256(static_cast<size_t>(BH) * L.nsplit * 4);
  L.off_cnt = L.off_part + round256(static_cast<size_t>(BH) * L.nsplit * d * 4);
  L.off_mr = L.off_cnt + round256(static_cast<size_t>(BH) * 4);
  L.total = L.off_mr + round256(static_cast<size_t>(BH) * 16);
  return L;
}

template <int D, bool kInt4 = false>
int decode_launch(const DecodeArgs& a, cudaStream_t stream) {
  const dim3 grid(a.nsplit, a.BH);
  if constexpr (kInt4) {
    intattn::decode::decode4_qk_kernel<D><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
  } else {
    if (a.k_u8)
      intattn::decode::decode_qk_kernel<D, true><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
    else
      intattn::decode::decode_qk_kernel<D, false><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
  }
  const int rc = note_launch(cudaGetLastError());
  if (rc != INTATTN_OK) return rc;
  if (kInt4 && a.nsplit == 1) {
    // one chunk per row: the P.V kernel computes m, Z and R itself
    intattn::decode::decode4_pv_kernel<D, true><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
    return note_launch(cudaGetLastError());
  }
  intattn::decode::decode_z_kernel<D><<<a.BH, intattn::decode::kThreads, 0, stream>>>(a);
  const int rz = note_launch(cudaGetLastError());
  if (rz != INTATTN_OK) return rz;
  if constexpr (kInt4) {
    intattn::decode::decode4_pv_kernel<D, false><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
  } else {
    if (a.v_u8)
      intattn::decode::decode_pv_kernel<D, true><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
    else
      intattn::decode::decode_pv_kernel<D, false><<<grid, intattn::decode::kThreads, 0, stream>>>(a);
  }
  return note_launch(cudaGetLastError());
}

// ------------------------------------------------------ failure self-test
// One CTA waits on an mbarrier that nothing will ever arrive on; the bounded
// wait gives up after its time limit and records the timeout in the device
// error word, exactly as a stalled pipeline role would.
__global__ void selftest_timeout_kernel() {
  __shared__ uint64_t bar;
  const uint32_t b = intattn::smem_u32(&bar);
  if (threadIdx.x == 0) {
    intattn::mbar_init(b, 1);
    intattn::mbar_fence_init();
  }
  __syncthreads();
  intattn::mbar_wait_warp(b, 0, 15u);
}

// ------------------------------------------------ static decode scratch
// Decode scratch for callers that cannot allocate device memory (see
// intattn_decode_static_scratch in intattn.h).  One array per GPU that loads
// this library, held until the process exits.  Host code must not pass the
// array's name to a kernel: on the host it is only a stand-in for the
// symbol, so its device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_decode_scratch[INTATTN_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[64] = {};

// Device address of g_decode_scratch on the current device (set up on the
// first call per device, with that device current).
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return note_launch(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return INTATTN_OK;
}

// Checks and kernel arguments shared by the decode entry points (the scratch
// is filled in by the caller of this helper).
int decode_setup(const int8_t* q, const int8_t* k_cache, const int8_t* v_cache, const intattn_scales_t* scales,
                 int B, int H, int Lk, int Lmax, int d, float clip_c, int8_t* out, DecodeArgs* a,
                 DecodeLayout* L, bool* empty, int chunk = intattn::decode::kChunk) {
  *empty = false;
  if (B < 0 || H <= 0 || Lk < 1 || Lk > 65535 || Lmax < Lk) return INTATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INTATTN_ERR_UNSUPPORTED;
  if (!scales) return INTATTN_ERR_INVALID_ARG;
  // kernel parameters up to 32764 bytes need CUDA 12.1 or later
  static_assert(sizeof(DecodeArgs) <= 8192, "kernel argument block too large");
  std::memset(a, 0, sizeof(*a));
  int rc = derive(scales, H, d, clip_c, a->lut, a->hp, INTATTN_MAX_HEADS);
  if (rc) return rc;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) {
    *empty = true;
    return INTATTN_OK;
  }
  if (BH > 65535) return INTATTN_ERR_UNSUPPORTED;  // grid y limit
  if (!q || !k_cache || !v_cache || !out) return INTATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return INTATTN_ERR_UNSUPPORTED;
  *L = decode_layout(BH, Lk, d, chunk);
  a->q = q;
  a->k = k_cache;
  a->v = v_cache;
  a->out = out;
  a->BH = static_cast<int32_t>(BH);
  a->H = H;
  a->Lk = Lk;
  a->Lmax = Lmax;
  a->nsplit = L->nsplit;
  a->ld_s = L->ld_s;
  a->chunk = chunk;
  a->per_head = scales->per_head ? 1 : 0;
  a->k_u8 = scales->z_k ? 1 : 0;
  a->v_u8 = scales->z_v ? 1 : 0;
  return INTATTN_OK;
}

void decode_scratch(DecodeArgs* a, const DecodeLayout& L, char* ws) {
  a->ws_s = reinterpret_cast<int32_t*>(ws + L.off_s);
  a->ws_max = reinterpret_cast<int32_t*>(ws + L.off_max);
  a->ws_part = reinterpret_cast<int32_t*>(ws + L.off_part);
  a->ws_cnt = reinterpret_cast<uint32_t*>(ws + L.off_cnt);  // zeroed by the first kernel of each call
  a->ws_mr = reinterpret_cast<int32_t*>(ws + L.off_mr);
}

}  // namespace

extern "C" {

int intattn_derive_params(const intattn_scales_t* scales, int H, int d, float clip_c, int32_t lut[32],
                          intattn_head_params_t* out) {
  if (!lut || !out) return INTATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INTATTN_ERR_UNSUPPORTED;
  uint32_t l[INTATTN_MAX_CLIPS][32];
  HeadParamsDev hp[INTATTN_MAX_HEADS];
  if (scales && !scales->per_head && H > 0) {
    // per-tensor: every head shares entry 0; any H is accepted
    const int rc = derive(scales, 1, d, clip_c, l, hp, INTATTN_MAX_HEADS);
    if (rc) return rc;
    for (int h = 0; h < H; ++h) out[h] = {hp[0].M, hp[0].s, hp[0].D, hp[0].Mo, hp[0].so};
  } else {
    const int rc = derive(scales, H, d, clip_c, l, hp, INTATTN_MAX_HEADS);
    if (rc) return rc;
    for (int h = 0; h < H; ++h) out[h] = {hp[h].M, hp[h].s, hp[h].D, hp[h].Mo, hp[h].so};
  }
  for (int i = 0; i < 32; ++i) lut[i] = static_cast<int32_t>(l[hp[0].lut][i]);
  return INTATTN_OK;
}

int intattn_forward(const int8_t* q, const int8_t* k, const int8_t* v, const intattn_scales_t* scales, int B,
                    int H, int Lq, int Lk, int d, int causal, float clip_c, int8_t* out,
                    intattn_stream_t stream) {
  return intattn_forward_variant(q, k, v, scales, B, H, Lq, Lk, d, causal, clip_c, out, INTATTN_VARIANT_AUTO,
                                 stream);
}

}  // extern "C"

namespace {

// The forward launch once the tables and head parameters are in `args`
// (args.lut, args.n_luts, args.per_head, and args.hp or args.hp_dev).
int forward_launch(const int8_t* q, const int8_t* k, const int8_t* v, PrefillArgs& args, int B, int H, int Lq,
                   int Lk, int d, int causal, int8_t* out, int variant, cudaStream_t st) {
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0 || Lq == 0) return INTATTN_OK;
  if (!q || !k || !v || !out) return INTATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return INTATTN_ERR_UNSUPPORTED;
  const int n_qtiles = (Lq + intattn::prefill::kBM - 1) / intattn::prefill::kBM;
  if (BH * n_qtiles > 0x7fffffffll || BH > 0x7fffffffll) return INTATTN_ERR_UNSUPPORTED;
  if (!encode_3d(&args.tm_q, q, d, Lq, BH, intattn::prefill::kBM) ||
      !encode_3d(&args.tm_k, k, d, Lk, BH, intattn::prefill::kBN) ||
      !encode_3d(&args.tm_v, v, d, Lk, BH, intattn::prefill::kBN))
    return INTATTN_ERR_CUDA;
  args.out = out;
  args.BH = static_cast<int32_t>(BH);
  args.H = H;
  args.Lq = Lq;
  args.Lk = Lk;
  args.causal = causal ? 1 : 0;
  args.n_qtiles = n_qtiles;
  args.n_tiles = static_cast<int32_t>(BH * n_qtiles);
  div_magic(static_cast<uint32_t>(BH), &args.div_bh_m, &args.div_bh_sh);
  div_magic(static_cast<uint32_t>(H), &args.div_h_m, &args.div_h_sh);
  int sms = 0;
  if (sm_count(&sms) != INTATTN_OK) return INTATTN_ERR_CUDA;
  // persistent kernel: one CTA per SM (each holds all 512 TMEM columns)
  const int grid = args.n_tiles < sms ? args.n_tiles : sms;
  // rows of at most 256 keys: the scores stay in tensor memory through the three sweeps
  const bool short_rows = variant == INTATTN_VARIANT_SHORT_ROWS ||
                          (variant == INTATTN_VARIANT_AUTO && Lk <= intattn::shortrow::kMaxKeys);
  if (short_rows)
    return args.v_u8 ? (d == 64 ? prefill_short_launch<64, true>(args, grid, st)
                                : prefill_short_launch<128, true>(args, grid, st))
                     : (d == 64 ? prefill_short_launch<64, false>(args, grid, st)
                                : prefill_short_launch<128, false>(args, grid, st));
  // the kernel instance with the V zero-point correction only when V has zero-points
  return args.v_u8 ? (d == 64 ? prefill_launch<64, true>(args, grid, st) : prefill_launch<128, true>(args, grid, st))
                   : (d == 64 ? prefill_launch<64, false>(args, grid, st) : prefill_launch<128, false>(args, grid, st));
}

// Exp tables of the distinct clip thresholds of n entries (clips[i], or
// clip_c for all when clips is null) and each entry's table index.
int clip_tables(const float* clips, float clip_c, int n, uint32_t lut[INTATTN_MAX_CLIPS][32], int32_t* idx,
                int* n_luts) {
  float seen[INTATTN_MAX_CLIPS];
  int m = 0;
  for (int i = 0; i < n; ++i) {
    const float c = clips ? clips[i] : clip_c;
    int id = 0;
    while (id < m && !(seen[id] == c)) ++id;
    if (id == m) {
      if (m == INTATTN_MAX_CLIPS) return INTATTN_ERR_UNSUPPORTED;
      const int rc = make_lut(static_cast<double>(c), lut[m]);
      if (rc) return rc;
      seen[m++] = c;
    }
    idx[i] = id;
  }
  *n_luts = m;
  return INTATTN_OK;
}

size_t align256_fp(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace of intattn_forward_fp: int8 q, k, v; the three scale arrays; the
// head parameters; the derivation status.
struct FpLayout {
  size_t q8, k8, v8, sc, zp, hp, status, total;
};

FpLayout fp_layout(int B, int H, int Lq, int Lk, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  FpLayout L{};
  L.q8 = 0;
  L.k8 = L.q8 + align256_fp(bh * Lq * d);
  L.v8 = L.k8 + align256_fp(bh * Lk * d);
  L.sc = L.v8 + align256_fp(bh * Lk * d);
  L.zp = L.sc + 3 * align256_fp(INTATTN_MAX_HEADS * sizeof(float));
  L.hp = L.zp + 2 * align256_fp(INTATTN_MAX_HEADS * sizeof(int32_t));
  L.status = L.hp + align256_fp(INTATTN_MAX_HEADS * sizeof(HeadParamsDev));
  L.total = L.status + 256;
  return L;
}

}  // namespace

extern "C" {

int intattn_forward_variant(const int8_t* q, const int8_t* k, const int8_t* v, const intattn_scales_t* scales,
                            int B, int H, int Lq, int Lk, int d, int causal, float clip_c, int8_t* out,
                            int variant, intattn_stream_t stream) {
  if (variant != INTATTN_VARIANT_AUTO && variant != INTATTN_VARIANT_THREE_PASS &&
      variant != INTATTN_VARIANT_SHORT_ROWS)
    return INTATTN_ERR_INVALID_ARG;
  if (variant == INTATTN_VARIANT_SHORT_ROWS && Lk > intattn::shortrow::kMaxKeys) return INTATTN_ERR_UNSUPPORTED;
  if (B < 0 || H <= 0 || Lq < 0 || Lk < 1 || Lk > 65535) return INTATTN_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return INTATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INTATTN_ERR_UNSUPPORTED;
  if (!scales) return INTATTN_ERR_INVALID_ARG;
  static_assert(sizeof(PrefillArgs) <= 8192, "kernel argument block too large");
  PrefillArgs args;
  std::memset(&args, 0, sizeof(args));
  int rc = derive(scales, H, d, clip_c, args.lut, args.hp, INTATTN_MAX_HEADS, &args.n_luts);
  if (rc) return rc;
  args.per_head = scales->per_head ? 1 : 0;
  args.k_u8 = scales->z_k ? 1 : 0;
  args.v_u8 = scales->z_v ? 1 : 0;
  return forward_launch(q, k, v, args, B, H, Lq, Lk, d, causal, out, variant, reinterpret_cast<cudaStream_t>(stream));
}

size_t intattn_forward_fp_workspace_size(int B, int H, int Lq, int Lk, int d) {
  if (B < 0 || H <= 0 || Lq < 0 || Lk < 1 || (d != 64 && d != 128)) return 0;
  return fp_layout(B, H, Lq, Lk, d).total;
}

}  // extern "C"

namespace {

int quantize_impl(const void* x, int dtype, int B, int H, int L, int d, int per_head, void* out, float* scales,
                  int32_t* zero_points, cudaStream_t st);

// intattn_forward_fp (asym_kv false) and intattn_forward_fp_zp (K and V
// quantised with zero-points, u8 codes).
int forward_fp_impl(const void* q, const void* k, const void* v, int dtype, int per_head, const float* s_o,
                    const float* clip, float clip_c, int B, int H, int Lq, int Lk, int d, int causal, int8_t* out,
                    float* scales_out, bool asym_kv, int32_t* zero_points_out, void* workspace,
                    size_t workspace_bytes, intattn_stream_t stream) {
  if (B < 0 || H <= 0 || Lq < 0 || Lk < 1 || Lk > 65535) return INTATTN_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return INTATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INTATTN_ERR_UNSUPPORTED;
  if (dtype != INTATTN_DTYPE_FP16 && dtype != INTATTN_DTYPE_BF16) return INTATTN_ERR_UNSUPPORTED;
  if (!s_o) return INTATTN_ERR_INVALID_ARG;
  const int n = per_head ? H : 1;
  if (n > INTATTN_MAX_HEADS) return INTATTN_ERR_UNSUPPORTED;
  static_assert(sizeof(intattn::DeriveArgs) <= 8192, "kernel argument block too large");
  intattn::DeriveArgs da;
  std::memset(&da, 0, sizeof(da));
  PrefillArgs args;
  std::memset(&args, 0, sizeof(args));
  int rc = clip_tables(clip, clip_c, n, args.lut, da.lut, &args.n_luts);
  if (rc) return rc;
  for (int i = 0; i < n; ++i) {
    const double so = s_o[i];
    if (!std::isfinite(so) || !(so > 0.0)) return INTATTN_ERR_PARAM_RANGE;
    da.s_o[i] = s_o[i];
    da.clip[i] = clip ? clip[i] : clip_c;
  }
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0 || Lq == 0) return INTATTN_OK;
  if (!q || !k || !v || !out) return INTATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return INTATTN_ERR_UNSUPPORTED;
  if (scales_out && (reinterpret_cast<uintptr_t>(scales_out) & 3u)) return INTATTN_ERR_UNSUPPORTED;
  if (zero_points_out && (reinterpret_cast<uintptr_t>(zero_points_out) & 3u)) return INTATTN_ERR_UNSUPPORTED;
  const FpLayout L = fp_layout(B, H, Lq, Lk, d);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return INTATTN_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  int8_t* q8 = reinterpret_cast<int8_t*>(ws + L.q8);
  int8_t* k8 = reinterpret_cast<int8_t*>(ws + L.k8);
  int8_t* v8 = reinterpret_cast<int8_t*>(ws + L.v8);
  float* sc = reinterpret_cast<float*>(ws + L.sc);
  const size_t sc_step = align256_fp(INTATTN_MAX_HEADS * sizeof(float)) / sizeof(float);
  float* s_q = sc;
  float* s_k = sc + sc_step;
  float* s_v = sc + 2 * sc_step;
  const size_t zp_step = align256_fp(INTATTN_MAX_HEADS * sizeof(int32_t)) / sizeof(int32_t);
  int32_t* z_k = asym_kv ? reinterpret_cast<int32_t*>(ws + L.zp) : nullptr;
  int32_t* z_v = asym_kv ? z_k + zp_step : nullptr;
  HeadParamsDev* hp = reinterpret_cast<HeadParamsDev*>(ws + L.hp);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  // quantise on the stream (scales stay on the device)
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((rc = quantize_impl(q, dtype, B, H, Lq, d, per_head, q8, s_q, nullptr, st)) ||
      (rc = quantize_impl(k, dtype, B, H, Lk, d, per_head, k8, s_k, z_k, st)) ||
      (rc = quantize_impl(v, dtype, B, H, Lk, d, per_head, v8, s_v, z_v, st)))
    return rc;
  da.s_q = s_q;
  da.s_k = s_k;
  da.s_v = s_v;
  da.z_v = z_v;
  da.hp = hp;
  da.status = status;
  da.n = n;
  da.d = d;
  intattn::params::derive_params_kernel<<<1, 128, 0, st>>>(da);
  if ((rc = note_launch(cudaGetLastError()))) return rc;
  if (scales_out) {
    for (int t = 0; t < 3; ++t)
      if ((rc = note_launch(cudaMemcpyAsync(scales_out + t * n, sc + t * sc_step, n * sizeof(float),
                                            cudaMemcpyDeviceToDevice, st))))
        return rc;
  }
  if (zero_points_out && asym_kv) {
    for (int t = 0; t < 2; ++t)
      if ((rc = note_launch(cudaMemcpyAsync(zero_points_out + t * n, z_k + t * zp_step, n * sizeof(int32_t),
                                            cudaMemcpyDeviceToDevice, st))))
        return rc;
  }
  args.per_head = per_head ? 1 : 0;
  args.k_u8 = asym_kv ? 1 : 0;
  args.v_u8 = asym_kv ? 1 : 0;
  args.hp_dev = hp;
  args.status = status;
  return forward_launch(q8, k8, v8, args, B, H, Lq, Lk, d, causal, out, INTATTN_VARIANT_AUTO, st);
}

}  // namespace

extern "C" {

int intattn_forward_fp(const void* q, const void* k, const void* v, int dtype, int per_head, const float* s_o,
                       const float* clip, float clip_c, int B, int H, int Lq, int Lk, int d, int causal,
                       int8_t* out, float* scales_out, void* workspace, size_t workspace_bytes,
                       intattn_stream_t stream) {
  return forward_fp_impl(q, k, v, dtype, per_head, s_o, clip, clip_c, B, H, Lq, Lk, d, causal, out, scales_out,
                         false, nullptr, workspace, workspace_bytes, stream);
}

int intattn_forward_fp_zp(const void* q, const void* k, const void* v, int dtype, int per_head, const float* s_o,
                          const float* clip, float clip_c, int B, int H, int Lq, int Lk, int d, int causal,
                          int8_t* out, float* scales_out, int32_t* zero_points_out, void* workspace,
                          size_t workspace_bytes, intattn_stream_t stream) {
  return forward_fp_impl(q, k, v, dtype, per_head, s_o, clip, clip_c, B, H, Lq, Lk, d, causal, out, scales_out,
                         true, zero_points_out, workspace, workspace_bytes, stream);
}

// ------------------------------------------------ forward from host buffers
namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// One workspace slot: device copies of q, k, v and out.
size_t host_slot_bytes(int B, int H, int Lq, int Lk, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t q = bh * Lq * d, kv = bh * Lk * d;
  return 2 * align256(q) + 2 * align256(kv);
}

// Two copy streams per device (host to device, device to host), created on
// first use and kept for the life of the process.
int copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  static std::mutex mu;
  static cudaStream_t streams[64][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev][0]) {
    cudaStream_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) return INTATTN_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(a);
      return INTATTN_ERR_CUDA;
    }
    streams[dev][0] = a;
    streams[dev][1] = b;
  }
  *h2d = streams[dev][0];
  *d2h = streams[dev][1];
  return INTATTN_OK;
}

// Per host thread and device, per workspace: which slot the next call takes
// and the events that order each slot's reuse (copied in, computed, copied
// out).  At most kMaxPipes workspaces are tracked; the least recently used
// one is retired once its events have completed (a host wait that only a
// thread cycling through more workspaces than that ever meets).
//
// Stream capture: a capture may not wait on an event recorded outside it
// (the dependency would cross the capture boundary), and an uncaptured call
// may not wait on an event recorded inside one.  Captured calls therefore
// record a separate set of events (cap_*) and wait on none recorded before
// the capture: each captured call forks its copy streams from `stream` and
// joins them back, so captured calls are ordered by `stream` alone.  Once a
// workspace has been used in a capture, the graph may be replayed on
// `stream` at any later point, so every later uncaptured call on that
// workspace also starts its copies after the work already on `stream`.
struct SlotEvents {
  cudaEvent_t in[2] = {}, done[2] = {}, out[2] = {};
  cudaEvent_t cap_in[2] = {}, cap_done[2] = {}, cap_out[2] = {};
  bool cap_events = false;  // cap_* created
  bool captured = false;    // used in a capture at least once
  int next = 0;
  unsigned long long used = 0;
};

struct HostPipes {
  cudaEvent_t fork = nullptr, cap_fork = nullptr;  // fork events outside and inside captures
  std::unordered_map<const void*, SlotEvents> by_ws;
  unsigned long long clock = 0;
};

constexpr size_t kMaxPipes = 64;

int make_events(SlotEvents* e) {
  cudaEvent_t* all[6] = {&e->in[0], &e->in[1], &e->done[0], &e->done[1], &e->out[0], &e->out[1]};
  for (cudaEvent_t* ev : all)
    if (cudaEventCreateWithFlags(ev, cudaEventDisableTiming) != cudaSuccess) return INTATTN_ERR_CUDA;
  return INTATTN_OK;
}

int make_capture_events(SlotEvents* e) {
  if (e->cap_events) return INTATTN_OK;
  cudaEvent_t* all[6] = {&e->cap_in[0], &e->cap_in[1], &e->cap_done[0], &e->cap_done[1], &e->cap_out[0],
                         &e->cap_out[1]};
  for (cudaEvent_t* ev : all)
    if (cudaEventCreateWithFlags(ev, cudaEventDisableTiming) != cudaSuccess) return INTATTN_ERR_CUDA;
  e->cap_events = true;
  return INTATTN_OK;
}

// The events of workspace `ws` for this thread and device (created on first
// use), and the fork event for a call inside (capturing) or outside a capture.
int pipe_of(const void* ws, bool capturing, cudaEvent_t* fork, SlotEvents** out) {
  thread_local HostPipes pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
  HostPipes& p = pipes[dev];
  cudaEvent_t& f = capturing ? p.cap_fork : p.fork;
  if (!f && cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess) return INTATTN_ERR_CUDA;
  auto it = p.by_ws.find(ws);
  if (it == p.by_ws.end()) {
    SlotEvents fresh;
    if (p.by_ws.size() >= kMaxPipes) {
      // retiring a workspace waits on the host, which a capture forbids
      if (capturing) return INTATTN_ERR_UNSUPPORTED;
      auto lru = p.by_ws.begin();
      for (auto i = p.by_ws.begin(); i != p.by_ws.end(); ++i)
        if (i->second.used < lru->second.used) lru = i;
      for (int sl = 0; sl < 2; ++sl)
        if (cudaEventSynchronize(lru->second.done[sl]) != cudaSuccess ||
            cudaEventSynchronize(lru->second.out[sl]) != cudaSuccess)
          return INTATTN_ERR_CUDA;
      fresh = lru->second;  // its events, now complete, serve the new workspace
      fresh.next = 0;
      fresh.captured = false;  // the new workspace has not been used in a capture
      p.by_ws.erase(lru);
    } else if (make_events(&fresh) != INTATTN_OK) {
      return INTATTN_ERR_CUDA;
    }
    it = p.by_ws.emplace(ws, fresh).first;
  }
  it->second.used = ++p.clock;
  *fork = f;
  *out = &it->second;
  return INTATTN_OK;
}

}  // namespace

size_t intattn_forward_host_workspace_size(int B, int H, int Lq, int Lk, int d) {
  if (B < 0 || H <= 0 || Lq < 0 || Lk < 1 || (d != 64 && d != 128)) return 0;
  return 2 * host_slot_bytes(B, H, Lq, Lk, d);
}

int intattn_forward_host(const int8_t* q, const int8_t* k, const int8_t* v, const intattn_scales_t* scales, int B,
                         int H, int Lq, int Lk, int d, int causal, float clip_c, int8_t* out, void* workspace,
                         size_t workspace_bytes, intattn_stream_t stream) {
  if (B < 0 || H <= 0 || Lq < 0 || Lk < 1 || Lk > 65535) return INTATTN_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return INTATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INTATTN_ERR_UNSUPPORTED;
  if (!scales) return INTATTN_ERR_INVALID_ARG;
  {
    // every parameter check of the forward, before anything is queued
    HeadParamsDev hp[INTATTN_MAX_HEADS];
    uint32_t l[INTATTN_MAX_CLIPS][32];
    const int rc = derive(scales, H, d, clip_c, l, hp, INTATTN_MAX_HEADS);
    if (rc) return rc;
  }
  if (static_cast<long long>(B) * H == 0 || Lq == 0) return INTATTN_OK;
  if (!q || !k || !v || !out) return INTATTN_ERR_INVALID_ARG;
  const size_t slot_bytes = host_slot_bytes(B, H, Lq, Lk, d);
  if (!workspace || workspace_bytes < 2 * slot_bytes) return INTATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return INTATTN_ERR_WORKSPACE;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream), h2d = nullptr, d2h = nullptr;
  cudaEvent_t e_fork = nullptr;
  SlotEvents* pipe = nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (note_launch(cudaStreamIsCapturing(st, &cap))) return INTATTN_ERR_CUDA;
  const bool capturing = cap != cudaStreamCaptureStatusNone;
  if (copy_streams(&h2d, &d2h)) return INTATTN_ERR_CUDA;
  if (const int prc = pipe_of(workspace, capturing, &e_fork, &pipe)) return prc;
  if (capturing && make_capture_events(pipe) != INTATTN_OK) return INTATTN_ERR_CUDA;
  const int sl = pipe->next;
  pipe->next = sl ^ 1;
  cudaEvent_t e_in = capturing ? pipe->cap_in[sl] : pipe->in[sl];
  cudaEvent_t e_done = capturing ? pipe->cap_done[sl] : pipe->done[sl];
  cudaEvent_t e_out = capturing ? pipe->cap_out[sl] : pipe->out[sl];
  if (capturing || pipe->captured) {
    // the copy streams start after the work already on `stream`: under
    // capture this is how they join the capture; after a capture, how they
    // wait for any replay of it
    if (note_launch(cudaEventRecord(e_fork, st)) || note_launch(cudaStreamWaitEvent(h2d, e_fork, 0)) ||
        note_launch(cudaStreamWaitEvent(d2h, e_fork, 0)))
      return INTATTN_ERR_CUDA;
  }
  // the slot's previous use: ordered by `stream` under capture (each
  // captured call ends joined to it), by the slot's events otherwise
  const bool wait_prev = !capturing;
  if (capturing) pipe->captured = true;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t qn = bh * Lq * d, kvn = bh * Lk * d;
  char* base = static_cast<char*>(workspace) + sl * slot_bytes;
  int8_t* dq = reinterpret_cast<int8_t*>(base);
  int8_t* dk = reinterpret_cast<int8_t*>(base + align256(qn));
  int8_t* dv = reinterpret_cast<int8_t*>(base + align256(qn) + align256(kvn));
  int8_t* dout = reinterpret_cast<int8_t*>(base + align256(qn) + 2 * align256(kvn));
  // copies in once this slot's previous forward has read its inputs; the
  // forward once they have landed and the slot's previous output has been
  // copied out; the copy out once the forward is done.  The copies of the
  // next call (other slot) overlap this call's forward and copy out.
  if ((wait_prev && note_launch(cudaStreamWaitEvent(h2d, e_done, 0))) ||
      note_launch(cudaMemcpyAsync(dq, q, qn, cudaMemcpyHostToDevice, h2d)) ||
      note_launch(cudaMemcpyAsync(dk, k, kvn, cudaMemcpyHostToDevice, h2d)) ||
      note_launch(cudaMemcpyAsync(dv, v, kvn, cudaMemcpyHostToDevice, h2d)) ||
      note_launch(cudaEventRecord(e_in, h2d)) || note_launch(cudaStreamWaitEvent(st, e_in, 0)) ||
      (wait_prev && note_launch(cudaStreamWaitEvent(st, e_out, 0))))
    return INTATTN_ERR_CUDA;
  const int rc = intattn_forward(dq, dk, dv, scales, B, H, Lq, Lk, d, causal, clip_c, dout, stream);
  if (rc) return rc;
  if (note_launch(cudaEventRecord(e_done, st)) || note_launch(cudaStreamWaitEvent(d2h, e_done, 0)) ||
      note_launch(cudaMemcpyAsync(out, dout, qn, cudaMemcpyDeviceToHost, d2h)) ||
      note_launch(cudaEventRecord(e_out, d2h)) || note_launch(cudaStreamWaitEvent(st, e_out, 0)))
    return INTATTN_ERR_CUDA;
  return INTATTN_OK;
}

size_t intattn_decode_workspace_size(int B, int H, int Lk, int d) {
  if (B < 0 || H <= 0 || Lk < 1 || (d != 64 && d != 128)) return 0;
  return decode_layout(static_cast<long long>(B) * H, Lk, d).total;
}

int intattn_decode(const int8_t* q, const int8_t* k_cache, const int8_t* v_cache, const intattn_scales_t* scales,
                   int B, int H, int Lk, int Lmax, int d, float clip_c, int8_t* out, void* workspace,
                   size_t workspace_bytes, intattn_stream_t stream) {
  DecodeArgs a;
  DecodeLayout L{};
  bool empty = false;
  int rc = decode_setup(q, k_cache, v_cache, scales, B, H, Lk, Lmax, d, clip_c, out, &a, &L, &empty);
  if (rc || empty) return rc;
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return INTATTN_ERR_WORKSPACE;
  decode_scratch(&a, L, static_cast<char*>(workspace));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? decode_launch<64>(a, st) : decode_launch<128>(a, st);
}

int intattn_decode_int4(const int8_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                        const intattn_scales_t* scales, int B, int H, int Lk, int Lmax, int d, float clip_c,
                        int8_t* out, void* workspace, size_t workspace_bytes, intattn_stream_t stream) {
  // unsigned int4 codes carry zero-points of 0 .. 15
  if (scales) {
    const int n = scales->per_head ? H : 1;
    for (int i = 0; scales->z_k && i < n && H > 0; ++i)
      if (scales->z_k[i] < 0 || scales->z_k[i] > 15) return INTATTN_ERR_INVALID_ARG;
    for (int i = 0; scales->z_v && i < n && H > 0; ++i)
      if (scales->z_v[i] < 0 || scales->z_v[i] > 15) return INTATTN_ERR_INVALID_ARG;
  }
  DecodeArgs a;
  DecodeLayout L{};
  bool empty = false;
  // fewer, longer splits than int8 (the per-CTA set-up and reduction are
  // amortised over more rows); the layout is never larger than the int8 one
  // that the workspace size query reports
  int rc = decode_setup(q, reinterpret_cast<const int8_t*>(k_cache), reinterpret_cast<const int8_t*>(v_cache),
                        scales, B, H, Lk, Lmax, d, clip_c, out, &a, &L, &empty, intattn::decode::kChunk4);
  if (rc || empty) return rc;
  // the documented requirement is intattn_decode_workspace_size (>= L.total)
  const size_t need = decode_layout(static_cast<long long>(B) * H, Lk, d).total;
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return INTATTN_ERR_WORKSPACE;
  decode_scratch(&a, L, static_cast<char*>(workspace));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? decode_launch<64, true>(a, st) : decode_launch<128, true>(a, st);
}

int intattn_decode_static_scratch(const int8_t* q, const int8_t* k_cache, const int8_t* v_cache,
                                  const intattn_scales_t* scales, int B, int H, int Lk, int Lmax, int d,
                                  float clip_c, int8_t* out, intattn_stream_t stream) {
  // same checks and kernels as intattn_decode; only the scratch differs
  DecodeArgs a;
  DecodeLayout L{};
  bool empty = false;
  int rc = decode_setup(q, k_cache, v_cache, scales, B, H, Lk, Lmax, d, clip_c, out, &a, &L, &empty);
  if (rc || empty) return rc;
  if (L.total > static_cast<size_t>(INTATTN_STATIC_SCRATCH_BYTES)) return INTATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  rc = static_scratch_address(&scratch);
  if (rc) return rc;
  decode_scratch(&a, L, static_cast<char*>(scratch));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? decode_launch<64>(a, st) : decode_launch<128>(a, st);
}

}  // extern "C"

namespace {

// intattn_quantize (zero_points == nullptr) and intattn_quantize_zp.
int quantize_impl(const void* x, int dtype, int B, int H, int L, int d, int per_head, void* out, float* scales,
                  int32_t* zero_points, cudaStream_t st) {
  if (B < 0 || H <= 0 || L < 0 || d <= 0) return INTATTN_ERR_INVALID_ARG;
  if (dtype != INTATTN_DTYPE_FP16 && dtype != INTATTN_DTYPE_BF16) return INTATTN_ERR_UNSUPPORTED;
  if (!scales) return INTATTN_ERR_INVALID_ARG;
  const long long slice = static_cast<long long>(L) * d;
  if (slice % intattn::quant::kVec) return INTATTN_ERR_UNSUPPORTED;  // whole 16-byte vectors per (b, h)
  if (reinterpret_cast<uintptr_t>(scales) & 3u) return INTATTN_ERR_UNSUPPORTED;
  if (zero_points && (reinterpret_cast<uintptr_t>(zero_points) & 3u)) return INTATTN_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  const int n_scales = per_head ? H : 1;
  uint32_t* nmax = reinterpret_cast<uint32_t*>(zero_points);
  if (BH == 0 || slice == 0) {
    // no elements: every scale is 1 (and every zero-point 0)
    intattn::quant::quant_scales_kernel<<<1, 128, 0, st>>>(reinterpret_cast<uint32_t*>(scales), nmax, n_scales);
    return note_launch(cudaGetLastError());
  }
  if (!x || !out) return INTATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return INTATTN_ERR_UNSUPPORTED;
  intattn::QuantArgs a;
  a.x = x;
  a.out = static_cast<int8_t*>(out);
  a.amax = reinterpret_cast<uint32_t*>(scales);
  a.nmax = nmax;
  a.asym = nmax ? 1 : 0;
  a.nvec = BH * (slice / intattn::quant::kVec);
  a.seg = per_head ? slice / intattn::quant::kVec : a.nvec;
  a.H = H;
  a.per_head = per_head ? 1 : 0;
  a.bf16 = dtype == INTATTN_DTYPE_BF16 ? 1 : 0;
  a.n_scales = n_scales;
  int sms = 0;
  if (sm_count(&sms) != INTATTN_OK) return INTATTN_ERR_CUDA;
  // one CTA per resident slot (the grid barrier needs them all resident),
  // each CTA >= one vector per thread
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, intattn::quant::quant_fused_kernel,
                                                    intattn::quant::kThreads, 0) != cudaSuccess || occ < 1)
    return note_launch(cudaGetLastError());
  const long long want = (a.nvec + intattn::quant::kThreads - 1) / intattn::quant::kThreads;
  const unsigned grid = static_cast<unsigned>(std::min<long long>(want, static_cast<long long>(sms) * occ));
  intattn::quant::quant_zero_kernel<<<1, 128, 0, st>>>(a.amax, a.nmax, n_scales, reinterpret_cast<uint32_t*>(out));
  const int rc = note_launch(cudaGetLastError());
  if (rc) return rc;
  // cooperative: all CTAs resident (the grid barrier); programmatic
  // serialisation: the loads of pass 1 overlap quant_zero
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(intattn::quant::kThreads);
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return note_launch(cudaLaunchKernelEx(&cfg, intattn::quant::quant_fused_kernel, a));
}

}  // namespace

extern "C" {

int intattn_quantize(const void* x, int dtype, int B, int H, int L, int d, int per_head, int8_t* out,
                     float* scales, intattn_stream_t stream) {
  return quantize_impl(x, dtype, B, H, L, d, per_head, out, scales, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int intattn_quantize_zp(const void* x, int dtype, int B, int H, int L, int d, int per_head, uint8_t* out,
                        float* scales, int32_t* zero_points, intattn_stream_t stream) {
  if (!zero_points) return INTATTN_ERR_INVALID_ARG;
  return quantize_impl(x, dtype, B, H, L, d, per_head, out, scales, zero_points,
                       reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Integer GELU parameters, IEEE double in the definition's order: index
// r = s_x 31 / (2c) as M / 2^s (M <= 2^24, s <= 26), the gate table
// G[i] = llround(2^15 Phi((2i - 31) c / 31)) with G[0] = 0 and G[31] = 2^15,
// and the requant m = s_x / (2^15 s_y) as Mo / 2^so.
int gelu_derive(float s_x_f, float s_y_f, float c_f, intattn_gelu_params_t* p) {
  const double s_x = s_x_f, s_y = s_y_f, c = c_f;
  if (!(std::isfinite(s_x) && s_x > 0.0 && std::isfinite(s_y) && s_y > 0.0 && std::isfinite(c) && c > 0.0))
    return INTATTN_ERR_PARAM_RANGE;
  const double r = (s_x * 31.0) / (2.0 * c);
  if (!(r < 1e15)) return INTATTN_ERR_PARAM_RANGE;  // M > 2^24 at every shift
  int sh = 26;
  while (sh > 1 && std::llround(std::ldexp(r, sh)) > (1LL << 24)) --sh;
  const long long M = std::llround(std::ldexp(r, sh));
  if (M < 1 || M > (1LL << 24)) return INTATTN_ERR_PARAM_RANGE;
  p->M = static_cast<int32_t>(M);
  p->s = sh;
  p->gate[0] = 0;
  p->gate[31] = 32768;
  for (int i = 1; i < 31; ++i) {
    const double t = (static_cast<double>(2 * i - 31) * c) / 31.0;
    p->gate[i] = static_cast<int32_t>(std::llround(32768.0 * (0.5 * std::erfc(-t / std::sqrt(2.0)))));
  }
  const double m = s_x / (32768.0 * s_y);
  int e = 0;
  const double f = std::frexp(m, &e);
  long long Mo = std::llround(f * 2147483648.0);
  if (Mo == (1LL << 31)) {
    Mo = 1LL << 30;
    ++e;
  }
  const int so = 31 - e;
  if (so < 1 || so > 62) return INTATTN_ERR_PARAM_RANGE;
  p->Mo = static_cast<int32_t>(Mo);
  p->so = so;
  return INTATTN_OK;
}

}  // namespace

int intattn_gelu_derive_params(float s_x, float s_y, float c, intattn_gelu_params_t* out) {
  if (!out) return INTATTN_ERR_INVALID_ARG;
  return gelu_derive(s_x, s_y, c, out);
}

int intattn_gelu(const int8_t* x, int8_t* y, long long n, float s_x, float s_y, float c, intattn_stream_t stream) {
  if (n < 0) return INTATTN_ERR_INVALID_ARG;
  intattn_gelu_params_t p;
  int rc = gelu_derive(s_x, s_y, c, &p);
  if (rc) return rc;
  if (n == 0) return INTATTN_OK;
  if (!x || !y) return INTATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return INTATTN_ERR_UNSUPPORTED;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
  if (xa != ya && xa < ya + static_cast<uintptr_t>(n) && ya < xa + static_cast<uintptr_t>(n))
    return INTATTN_ERR_INVALID_ARG;  // partial overlap (in place is fine)
  intattn::GeluArgs a;
  a.x = x;
  a.y = y;
  a.n = n;
  a.M = p.M;
  a.s = p.s;
  a.Mo = p.Mo;
  a.so = p.so;
  for (int i = 0; i < 32; ++i) a.gate[i] = p.gate[i];
  int sms = 0;
  if (sm_count(&sms) != INTATTN_OK) return INTATTN_ERR_CUDA;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, intattn::gelu::gelu_kernel, intattn::gelu::kThreads, 0) !=
          cudaSuccess ||
      occ < 1)
    return note_launch(cudaGetLastError());
  const long long per_cta = static_cast<long long>(intattn::gelu::kThreads) * intattn::gelu::kBatch;
  const long long want = std::max(1LL, ((n >> 4) + per_cta - 1) / per_cta);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(want, static_cast<long long>(sms) * occ));
  intattn::gelu::gelu_kernel<<<grid, intattn::gelu::kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return note_launch(cudaGetLastError());
}

size_t intattn_calibrate_workspace_size(int B, int H) {
  if (B < 0 || H <= 0) return 0;
  return (static_cast<size_t>(B) * H * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
}

int intattn_calibrate_clip(const int8_t* q, const int8_t* k, const intattn_scales_t* scales, int B, int H, int Lq,
                           int Lk, int d, int causal, int keep, int stride, float c_min, float c_max, float* clip_out,
                           int32_t* gaps_out, void* workspace, size_t workspace_bytes, intattn_stream_t stream) {
  if (B < 0 || H <= 0 || Lq < 0 || Lk < 1 || Lk > 65535 || keep < 1 || stride < 1) return INTATTN_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return INTATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INTATTN_ERR_UNSUPPORTED;
  if (!scales || !scales->s_q || !scales->s_k || !clip_out) return INTATTN_ERR_INVALID_ARG;
  if (scales->z_k || scales->z_v) return INTATTN_ERR_UNSUPPORTED;  // int8 codes only
  if (!std::isfinite(c_min) || !std::isfinite(c_max) || !(c_min > 0.0f) || !(c_max >= c_min))
    return INTATTN_ERR_PARAM_RANGE;
  const int n = scales->per_head ? H : 1;
  for (int i = 0; i < n; ++i)
    if (!std::isfinite(scales->s_q[i]) || !std::isfinite(scales->s_k[i]) || !(scales->s_q[i] > 0.0f) ||
        !(scales->s_k[i] > 0.0f))
      return INTATTN_ERR_PARAM_RANGE;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 65535) return INTATTN_ERR_UNSUPPORTED;  // grid y
  std::vector<int32_t> G(static_cast<size_t>(BH), 0);
  const int rows = Lq / stride;  // sampled rows stride - 1, 2 stride - 1, ...
  if (BH > 0 && rows > 0) {
    if (!q || !k) return INTATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k)) return INTATTN_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < intattn_calibrate_workspace_size(B, H) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return INTATTN_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t* dG = static_cast<int32_t*>(workspace);
    intattn::CalibArgs a{q, k, dG, Lq, Lk, d, causal ? 1 : 0, keep, stride};
    int rc = note_launch(cudaMemsetAsync(dG, 0, static_cast<size_t>(BH) * sizeof(int32_t), st));
    if (rc) return rc;
    // scores computed once per sampled row, in shared memory, while a CTA's
    // rows fit; else recomputed in each radix pass
    const int per_cta = static_cast<int>(std::min<long long>(
        intattn::calib::kRowsMax, (200ll * 1024) / (4ll * (((Lk + 3) & ~3)))));
    if (per_cta >= 1) {
      const size_t smem = static_cast<size_t>(per_cta) * (((Lk + 3) & ~3)) * 4;
      static bool attr_set[64] = {};
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return INTATTN_ERR_CUDA;
      if (!attr_set[dev]) {
        if ((rc = note_launch(cudaFuncSetAttribute(intattn::calib::gap_rows_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024))))
          return rc;
        attr_set[dev] = true;
      }
      const unsigned blocks = static_cast<unsigned>((rows + per_cta - 1) / per_cta);
      intattn::calib::gap_rows_kernel<<<dim3(blocks, static_cast<unsigned>(BH)), intattn::calib::kRowsThreads, smem,
                                        st>>>(a, per_cta, rows);
    } else {
      intattn::calib::gap_kernel<<<dim3(rows, static_cast<unsigned>(BH)), intattn::calib::kThreads, 0, st>>>(a);
    }
    if ((rc = note_launch(cudaGetLastError()))) return rc;
    if ((rc = note_launch(cudaMemcpyAsync(G.data(), dG, G.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, st))))
      return rc;
    if ((rc = note_launch(cudaStreamSynchronize(st)))) return rc;
  }
  // the threshold of each entry from its largest gap, IEEE double in this order
  for (int e = 0; e < n; ++e) {
    int32_t g = 0;
    for (long long bh = 0; bh < BH; ++bh)
      if (!scales->per_head || bh % H == e) g = std::max(g, G[static_cast<size_t>(bh)]);
    const double alpha = (static_cast<double>(scales->s_q[e]) * static_cast<double>(scales->s_k[e])) /
                         std::sqrt(static_cast<double>(d));
    const double c = ((alpha * static_cast<double>(g)) * 31.0) / 30.0;
    clip_out[e] = static_cast<float>(std::min(std::max(c, static_cast<double>(c_min)), static_cast<double>(c_max)));
    if (gaps_out) gaps_out[e] = g;
  }
  return INTATTN_OK;
}

int intattn_selftest_timeout(intattn_stream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return note_launch(cudaGetLastError());
}

int intattn_device_error(intattn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return INTATTN_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, intattn::g_device_error, sizeof(v)) != cudaSuccess) return INTATTN_ERR_CUDA;
  if (v == 0) return INTATTN_OK;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(intattn::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return INTATTN_ERR_CUDA;
  return (v & intattn::kErrTimeout) ? INTATTN_ERR_TIMEOUT : INTATTN_ERR_PARAM_RANGE;
}

const char* intattn_strerror(int code) {
  switch (code) {
    case INTATTN_OK: return "ok";
    case INTATTN_ERR_INVALID_ARG: return "invalid argument";
    case INTATTN_ERR_UNSUPPORTED: return "unsupported shape, alignment or head count";
    case INTATTN_ERR_PARAM_RANGE: return "scale or clip out of range";
    case INTATTN_ERR_CUDA:
      return g_last_cuda_error ? g_last_cuda_error : "CUDA launch or driver call failed";
    case INTATTN_ERR_WORKSPACE: return "decode workspace missing, misaligned or too small";
    case INTATTN_ERR_TIMEOUT: return "a kernel wait timed out";
    default: return "unknown error";
  }
}

}  // extern "C"
