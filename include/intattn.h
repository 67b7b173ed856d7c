/*
 * intattn.h -- C ABI of the B200 (sm_100a) fully-integer attention forward.
 *
 * Method: IntAttention (arXiv 2511.21513), as summarised on the euno.news
 * pages "IntAttention: a fully-integer attention pipeline for efficient edge
 * inference" (Chinese and Korean editions), section "Methodology":
 *   item 2  IndexSoftmax -- the int32 attention scores are clipped by a
 *           sparsity-aware threshold, looked up in a 32-entry exp table, the
 *           looked-up pseudo-exponentials are summed in int32 and scaled by a
 *           reciprocal with an integer multiply and a right shift;
 *   item 3  Q.K^T and V.softmax stay in the integer domain (end-to-end INT8).
 * The pages fix no constant, rounding rule or width.  The exact definition
 * this library computes (identical, bit for bit, to the CPU oracle that the
 * tests compare it with) is:
 *
 *   per head h:  alpha = s_q s_k / sqrt(d);  r = alpha * 31 / c
 *                s = 26, lowered while llround(r 2^s) > 2^24;  M = llround(r 2^s)
 *                D = ceil(61 2^(s-1) / M)   (smallest gap with index 31)
 *                LUT[i] = llround(2^15 exp(-i c / 31)), i < 31;  LUT[31] = 0
 *                s_v / (255 s_o) = f 2^e, f in [0.5,1):  Mo = llround(f 2^31),
 *                so = 31 - e  (Mo == 2^31 -> Mo = 2^30, so - 1)
 *   per row i:   S_j = sum_t Q[i,t] K[j,t] over valid keys j (causal: j <= i + Lk - Lq)
 *                m = max_j S_j;  idx_j = (min(m - S_j, D) M + 2^(s-1)) >> s
 *                E_j = LUT[idx_j];  Z = sum_j E_j  (int32)
 *                R = floor((255 2^32 + floor(Z/2)) / Z)
 *                P_j = (E_j R + 2^31) >> 32        (u8, sums to about 255)
 *                acc_t = sum_j P_j V[j,t]          (int32)
 *                out_t = clamp((acc_t Mo + 2^(so-1)) >> so, -127, 127)  (floor shift)
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers, 16-byte aligned, row-major and
 *     contiguous with the innermost dimension d.  The caller owns them.
 *   - The library allocates and frees nothing, never synchronises the stream
 *     (except intattn_device_error and intattn_calibrate_clip, which return
 *     results to the host), and launches only on the given stream.
 *     Calls are asynchronous: a 0 return means the work was enqueued.
 *     One exception: intattn_forward_host (host buffers) creates two copy
 *     streams per device and events per workspace on first use, runs its
 *     copies on those streams, and can wait on the host when a host thread
 *     cycles through more than 64 workspaces (see its comment).
 *   - Scale arrays are HOST pointers, read during the call only.
 *   - d must be 64 or 128; 1 <= Lk <= 65535 (keeps Z < 2^31).
 *   - Return codes are the INTATTN_* values below; on any non-zero return
 *     nothing was launched (INTATTN_ERR_CUDA: a launch was refused).
 */
#ifndef INTATTN_H
#define INTATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without requiring the CUDA headers (same underlying type). */
typedef struct CUstream_st *intattn_stream_t;

enum {
    INTATTN_OK = 0,
    INTATTN_ERR_INVALID_ARG = 1,  /* null pointer, negative size, causal with Lq > Lk, Lk out of range */
    INTATTN_ERR_UNSUPPORTED = 2,  /* d not 64/128, misaligned pointer, too many heads */
    INTATTN_ERR_PARAM_RANGE = 3,  /* scale or clip not finite / not > 0; M or so out of range */
    INTATTN_ERR_CUDA = 4,         /* a CUDA launch or driver call failed */
    INTATTN_ERR_WORKSPACE = 5,    /* decode workspace missing or too small */
    INTATTN_ERR_TIMEOUT = 6       /* a kernel wait ran out (reported by intattn_device_error) */
};

/* Largest H for per-head scales (the per-head parameters travel as kernel
 * arguments). */
#define INTATTN_MAX_HEADS 128

/* Quantisation scales (real value = scale * int8 code).  per_head = 0: each
 * array holds one entry shared by all heads; per_head = 1: H entries.
 * clip_c (optional): per-head clip thresholds in the same layout (the
 * authors name a learned / adaptive clip as future work: this is where a
 * calibrated threshold per head goes in); NULL: the clip_c argument of the
 * call applies to every head.  At most INTATTN_MAX_CLIPS distinct values per
 * call (each needs its own exp table), else INTATTN_ERR_UNSUPPORTED. */
typedef struct intattn_scales {
    int32_t per_head;
    const float *s_q;
    const float *s_k;
    const float *s_v;
    const float *s_o;
    const float *clip_c;
    /* Zero-points (optional, host, the layout of the scales), the forum page's
     * dynamic scale and zero-point (section 动态量化策略): z_k != NULL means the K
     * codes are u8 (the k / k_cache pointer is read as uint8_t) and code c
     * stands for c - z_k; likewise z_v for V.  Each zero-point is 0 .. 255,
     * else INTATTN_ERR_INVALID_ARG.  The definition then reads
     * S_j = sum_t Q[i,t] (K[j,t] - z_k) and acc_t = sum_j P_j (V[j,t] - z_v).
     * Q stays symmetric int8.  Accepted by the forward, intattn_forward_variant,
     * intattn_forward_host and both decodes (intattn_decode_int4: unsigned
     * nibbles c in [0, 15] with zero-points 0 .. 15 instead of two's complement
     * nibbles); intattn_calibrate_clip returns INTATTN_ERR_UNSUPPORTED. */
    const int32_t *z_k;
    const int32_t *z_v;
} intattn_scales_t;

#define INTATTN_MAX_CLIPS 8

/* Derived integer parameters of one head (see the definition above). */
typedef struct intattn_head_params {
    int32_t M;   /* index multiplier            */
    int32_t s;   /* index shift, 1..26          */
    int32_t D;   /* gap clip                    */
    int32_t Mo;  /* requantisation multiplier   */
    int32_t so;  /* requantisation shift, 1..62 */
} intattn_head_params_t;

/* Host-only: derive the LUT and the per-head parameters exactly as the
 * kernels use them.  lut: 32 entries (the table of head 0's clip threshold);
 * out: H entries.  No GPU needed. */
int intattn_derive_params(const intattn_scales_t *scales, int H, int d, float clip_c,
                          int32_t lut[32], intattn_head_params_t *out);

/* Prefill / full forward (IntAttention "Methodology" items 2-3).
 *   q   [B, H, Lq, d] int8      k, v [B, H, Lk, d] int8      out [B, H, Lq, d] int8
 *   causal != 0: key j is visible to query i iff j <= i + (Lk - Lq) (requires Lq <= Lk).
 *   clip_c: the sparsity-aware clip threshold, in logit units (> 0).
 * B*H*Lq == 0 returns INTATTN_OK without a launch. */
int intattn_forward(const int8_t *q, const int8_t *k, const int8_t *v,
                    const intattn_scales_t *scales, int B, int H, int Lq, int Lk, int d,
                    int causal, float clip_c, int8_t *out, intattn_stream_t stream);

/* Kernel choice of intattn_forward_variant. */
enum {
    INTATTN_VARIANT_AUTO = 0,        /* what intattn_forward does: SHORT_ROWS when Lk <= 256, else THREE_PASS */
    INTATTN_VARIANT_THREE_PASS = 1,  /* scores recomputed by the tensor core in each of the three sweeps */
    INTATTN_VARIANT_SHORT_ROWS = 2   /* Lk <= 256: the scores of a 128-row tile stay in tensor memory through
                                        all three sweeps (one Q.K^T per key tile) */
};

/* intattn_forward with an explicit kernel choice (for measuring the
 * variants against each other; every variant computes the same bytes).
 * SHORT_ROWS with Lk > 256 returns INTATTN_ERR_UNSUPPORTED; an unknown
 * variant INTATTN_ERR_INVALID_ARG.  Otherwise as intattn_forward. */
int intattn_forward_variant(const int8_t *q, const int8_t *k, const int8_t *v,
                            const intattn_scales_t *scales, int B, int H, int Lq, int Lk, int d,
                            int causal, float clip_c, int8_t *out, int variant, intattn_stream_t stream);

/* Bytes of device workspace intattn_forward_host needs for these sizes
 * (0 for invalid sizes). */
size_t intattn_forward_host_workspace_size(int B, int H, int Lq, int Lk, int d);

/* intattn_forward on HOST tensors: q, k, v and out are host pointers in the
 * layout of intattn_forward; page-locked (pinned) memory lets the copies run
 * asynchronously, pageable memory works but the copies then serialise with
 * the host.  The inputs are copied in on a library copy stream, the forward
 * runs on `stream`, the output is copied out on a second copy stream.  The
 * workspace has two slots that consecutive calls with the same workspace
 * from one host thread alternate between, so the copies in of one call
 * overlap the forward and the copy out of the previous one: a sequence of
 * calls costs about the host-to-device copy time per call.
 *   workspace: device, 256-byte aligned, at least
 *   intattn_forward_host_workspace_size(B, H, Lq, Lk, d) bytes (two slots of
 *   q, k, v and out); contents need no initialisation.  Calls that share a
 *   workspace must come from one host thread.
 * The library keeps two copy streams per device (created on first use, kept
 * for the process) and, per host thread and device, six events for each of
 * up to 64 workspaces (a 65th workspace waits on the host for the least
 * recently used one's copies to finish and takes its events).  The result
 * is in `out` when `stream` reaches the end of the call; q, k, v and out must
 * stay valid and unmodified until then.
 * Stream capture: a captured call forks its copy streams from `stream` and
 * joins them back; it records its own set of events and waits on no event
 * recorded outside the capture, so captured calls are ordered by `stream`
 * alone and do not overlap each other.  Replays of the graph must be
 * ordered on `stream` with other calls on the same workspace.  After a
 * workspace has been used in a capture, later uncaptured calls on it also
 * start their copies after the work already on `stream` (a replay may be
 * there), so they no longer overlap each other: give captured and uncaptured
 * calls separate workspaces to keep the uncaptured ones overlapped.  A capture that would
 * need a 65th workspace returns INTATTN_ERR_UNSUPPORTED.  Return codes as
 * intattn_forward, plus INTATTN_ERR_WORKSPACE. */
int intattn_forward_host(const int8_t *q, const int8_t *k, const int8_t *v,
                         const intattn_scales_t *scales, int B, int H, int Lq, int Lk, int d,
                         int causal, float clip_c, int8_t *out, void *workspace,
                         size_t workspace_bytes, intattn_stream_t stream);

/* Bytes of device workspace intattn_decode needs for these sizes. */
size_t intattn_decode_workspace_size(int B, int H, int Lk, int d);

/* Decode: one query per (b, h) against the first Lk rows of an int8 KV cache
 * of capacity Lmax rows (same definition with Lq = 1, no mask).
 *   q [B, H, 1, d]   k_cache, v_cache [B, H, Lmax, d]   out [B, H, 1, d]
 *   workspace: caller-owned device buffer of at least
 *   intattn_decode_workspace_size(B, H, Lk, d) bytes, 256-byte aligned; its
 *   contents need no initialisation and are overwritten.  Calls that share a
 *   workspace must be ordered on one stream. */
int intattn_decode(const int8_t *q, const int8_t *k_cache, const int8_t *v_cache,
                   const intattn_scales_t *scales, int B, int H, int Lk, int Lmax, int d,
                   float clip_c, int8_t *out, void *workspace, size_t workspace_bytes,
                   intattn_stream_t stream);

/* Decode over an int4 KV cache (IntAttention Methodology item 3 with 4-bit
 * keys and values: the same integer definition, with K and V codes in
 * [-8, 7] and s_k, s_v the scales of those codes).  Halves the bytes a
 * decode step streams.
 *   k_cache, v_cache: [B, H, Lmax, d/2] bytes; byte t of a row holds channel
 *   2t in bits 0-3 and channel 2t+1 in bits 4-7, each a 4-bit two's
 *   complement value.  q [B, H, 1, d] int8, out [B, H, 1, d] int8.
 *   Workspace: as intattn_decode (intattn_decode_workspace_size).
 *   Arguments, contracts and return codes: as intattn_decode. */
int intattn_decode_int4(const int8_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                        const intattn_scales_t *scales, int B, int H, int Lk, int Lmax, int d,
                        float clip_c, int8_t *out, void *workspace, size_t workspace_bytes,
                        intattn_stream_t stream);

/* Element types accepted by intattn_quantize. */
enum { INTATTN_DTYPE_FP16 = 0, INTATTN_DTYPE_BF16 = 1 };

/* Quantisation prologue (the step upstream of the integer pipeline: the
 * forum page "IntAttention：面向边缘设备的纯整数注意力推理加速方案", section
 * 动态量化策略, sets each layer's or head's range from the live activations).
 *   x   [B, H, L, d] fp16 or bf16 (dtype), device, 16-byte aligned
 *   out [B, H, L, d] int8 codes, device, 16-byte aligned, not overlapping
 *   x; its first 8 bytes hold two grid-barrier counters until the call ends
 *   scales: DEVICE float buffer of H entries (per_head) or 1, overwritten
 *   with the scales (real value = scale * code); holds amax meanwhile.
 * Definition: amax = max |x| over the tensor (or over head h);
 *   s = amax / 127 and inv = min(127 / amax, FLT_MAX) in IEEE fp32 (both 1
 *   when amax = 0);
 *   code = clamp(rint(x * inv), -127, 127), fp32 product rounded to
 *   nearest, rint half to even.  Symmetric: zero-point 0.  Inputs must be
 *   finite.
 * L * d must be a multiple of 8.  Asynchronous on `stream`; the scales are on
 * the device when the stream reaches the end of the call (a caller that
 * passes them to intattn_forward reads them back first).
 * B*H*L*d == 0 only sets the scales to 1.
 * Two launches: a zeroing kernel and one cooperative single-pass kernel
 * (max |x|, a bounded grid barrier, codes); a barrier that times out is
 * reported by intattn_device_error. */
int intattn_quantize(const void *x, int dtype, int B, int H, int L, int d, int per_head, int8_t *out,
                     float *scales, intattn_stream_t stream);

/* Asymmetric quantisation prologue: the zero-point the same page names beside
 * the scale.  u8 codes and a zero-point per tensor or head:
 *   hi = max(max x, 0), lo = min(min x, 0) over the tensor (or head h) -- the
 *   range always holds 0, so 0 is the code z;
 *   w = hi - lo in IEEE double; s = RN32(w / 255) and inv = RN32(min(255 / w,
 *   FLT_MAX)) (both 1 when w = 0);
 *   z = clamp(rint(RN32(-lo * inv)), 0, 255);
 *   code = clamp(rint(RN32(x * inv)) + z, 0, 255), rint half to even.
 * A code c stands for s * (c - z).
 *   out [B, H, L, d] u8 codes (first 8 bytes: barrier counters until the end)
 *   scales: DEVICE float [H] or [1]; zero_points: DEVICE int32 [H] or [1]
 *   (holds the bits of max(-lo) until the end).  Everything else as
 *   intattn_quantize; INVALID_ARG for zero_points == NULL. */
int intattn_quantize_zp(const void *x, int dtype, int B, int H, int L, int d, int per_head, uint8_t *out,
                        float *scales, int32_t *zero_points, intattn_stream_t stream);

/* Bytes of device workspace intattn_forward_fp needs for these sizes (0 for
 * invalid sizes): int8 copies of q, k and v, three scale arrays, the head
 * parameters and a status word. */
size_t intattn_forward_fp_workspace_size(int B, int H, int Lq, int Lk, int d);

/* The forward from fp16 / bf16 activations, with no host round trip: the
 * quantisation prologue above (the forum page's 动态量化策略: each tensor's, or
 * each head's, scale taken from the live activations) runs on q, k and v into
 * the workspace; a one-CTA kernel derives every head's integer parameters on
 * the device from those scales, in the same IEEE double steps as
 * intattn_derive_params (so they are identical); the integer forward then
 * reads them from device memory.  The result equals quantising each tensor
 * with intattn_quantize and calling intattn_forward with the resulting scales.
 *   q [B, H, Lq, d], k, v [B, H, Lk, d]: device, dtype INTATTN_DTYPE_FP16 or
 *   INTATTN_DTYPE_BF16, 16-byte aligned, finite values.
 *   per_head: scales per head (1) or per tensor (0), for q, k and v alike.
 *   s_o: HOST, the output scale (H entries per head, or 1).
 *   clip: HOST per-entry clip thresholds in the layout of s_o, or NULL for
 *   clip_c everywhere (at most INTATTN_MAX_CLIPS distinct values).
 *   out [B, H, Lq, d] int8, device.
 *   scales_out: NULL, or DEVICE floats receiving s_q, s_k, s_v (each H or 1
 *   entries, in that order) for the caller's own use.
 *   workspace: device, 256-byte aligned, at least
 *   intattn_forward_fp_workspace_size bytes; calls that share it must be
 *   ordered on one stream.
 * A derived parameter out of range (see intattn_derive_params) cannot be
 * reported by the return code, since the scales are only known on the
 * device: the forward then writes nothing, and intattn_device_error returns
 * INTATTN_ERR_PARAM_RANGE.  Launches: 2 per tensor (quantisation), 1
 * (parameters), 1 (forward).  Return codes as intattn_forward, plus
 * INTATTN_ERR_WORKSPACE. */
int intattn_forward_fp(const void *q, const void *k, const void *v, int dtype, int per_head,
                       const float *s_o, const float *clip, float clip_c, int B, int H, int Lq, int Lk,
                       int d, int causal, int8_t *out, float *scales_out, void *workspace,
                       size_t workspace_bytes, intattn_stream_t stream);

/* intattn_forward_fp with K and V quantised with zero-points (u8 codes, the
 * rule of intattn_quantize_zp) and Q symmetric, then the integer forward
 * with those zero-points (the definition under intattn_scales_t.z_k / z_v).
 * zero_points_out (optional, DEVICE int32, 4-byte aligned): receives z_k then
 * z_v (H entries each per head, else one each).  Workspace, arguments and
 * return codes as intattn_forward_fp. */
int intattn_forward_fp_zp(const void *q, const void *k, const void *v, int dtype, int per_head, const float *s_o,
                          const float *clip, float clip_c, int B, int H, int Lq, int Lk, int d, int causal,
                          int8_t *out, float *scales_out, int32_t *zero_points_out, void *workspace,
                          size_t workspace_bytes, intattn_stream_t stream);

/* Bytes of device workspace intattn_calibrate_clip needs (0 for invalid sizes). */
size_t intattn_calibrate_workspace_size(int B, int H);

/* Adaptive clip thresholds from the scores themselves.  The summary pages
 * (sections 概览 / Overview and 局限性与未来工作 / Limitations & Future Work)
 * describe the clip as sparsity-aware, limiting extreme activations
 * dynamically, and name an adaptive threshold as future work without a rule;
 * this is the library's reading:
 *   sampled rows i = stride - 1, 2 stride - 1, ... < Lq of every (b, h);
 *   G_i = m_i - S_i,(K): the gap from the row max to the K-th largest score
 *   (K = keep) over the row's valid keys (causal as intattn_forward), or to
 *   the smallest score when fewer than K keys are valid;
 *   G = max of G_i over the sampled rows and the batch (per head), or over
 *   everything (per-tensor scales);
 *   c = clamp(alpha G 31 / 30, c_min, c_max), alpha = s_q s_k / sqrt(d), in
 *   IEEE double in that order, then rounded to float.
 * Every sampled row then keeps at least K keys at a table index <= 30
 * (unclipped), with the threshold, and so the table spacing c / 31, as small
 * as that allows.  The result goes to the clip_c member of intattn_scales_t.
 *   q [B, H, Lq, d], k [B, H, Lk, d]: device int8.  scales: HOST, s_q and s_k
 *   used (per_head as given).  clip_out: HOST, H entries per head or 1.
 *   gaps_out: NULL or HOST, the same count: the integer G of each entry.
 *   workspace: device, 256-byte aligned, intattn_calibrate_workspace_size.
 * Unlike the other entry points this one returns its result to the host, so
 * it synchronises `stream` before returning (one kernel launch, one copy). */
int intattn_calibrate_clip(const int8_t *q, const int8_t *k, const intattn_scales_t *scales, int B, int H,
                           int Lq, int Lk, int d, int causal, int keep, int stride, float c_min, float c_max,
                           float *clip_out, int32_t *gaps_out, void *workspace, size_t workspace_bytes,
                           intattn_stream_t stream);

/* Integer GELU (the summary page "[Paper] IntAttention：全整数注意力流水线用于
 * 高效边缘推理", section 局限性与未来工作, names GELU as the next operator for the
 * method; this definition is the library's reading of "the same machinery":
 * an index by integer multiply and shift, a 32-entry integer gate table, a
 * requantising multiply and shift).  Real values: x = s_x * q, y = s_y * out.
 *   r = (s_x * 31) / (2c); s = 26, lowered while llround(r 2^s) > 2^24;
 *   M = llround(r 2^s) in [1, 2^24]
 *   gate[i] = llround(32768 * (0.5 * erfc(-t_i / sqrt 2))), t_i = ((2i - 31) c) / 31,
 *   i = 1..30; gate[0] = 0, gate[31] = 32768
 *   m = s_x / (32768 s_y) = f 2^e; Mo = llround(f 2^31) (2^31 -> 2^30, e+1);
 *   so = 31 - e in [1, 62]
 *   per element: idx = clamp(16 + floor(q M / 2^s), 0, 31); y = q * gate[idx];
 *   out = clamp(floor((y Mo + 2^(so-1)) / 2^so), -127, 127)
 * (IEEE double in that order; llround rounds half away from zero.) */
typedef struct {
    int32_t M, s;       /* index multiplier and shift */
    int32_t Mo, so;     /* requant multiplier and shift */
    int32_t gate[32];   /* 2^15 * Phi at the 32 table points */
} intattn_gelu_params_t;

/* Host only: the parameters above.  PARAM_RANGE for a scale or c that is not
 * finite and > 0, or M / so out of range; INVALID_ARG for out == NULL. */
int intattn_gelu_derive_params(float s_x, float s_y, float c, intattn_gelu_params_t *out);

/* y[i] = integer GELU of x[i], i < n.  x, y: device, 16-byte aligned; y == x
 * (in place) is allowed, any other overlap is INVALID_ARG.  n == 0 launches
 * nothing.  One launch, asynchronous on `stream`. */
int intattn_gelu(const int8_t *x, int8_t *y, long long n, float s_x, float s_y, float c,
                 intattn_stream_t stream);

/* Capacity in bytes of the library's static decode scratch (48 MiB). */
#define INTATTN_STATIC_SCRATCH_BYTES (48u * 1024u * 1024u)

/* Decode without any allocation: intattn_decode with the scratch taken from a
 * fixed array inside this library instead of a caller workspace.  The paper
 * has no counterpart; it exists for callers that cannot allocate device
 * memory on their call path -- for example a plugin that runs under a host
 * framework's own caching allocator and has no workspace to hand over, or a
 * latency-bound serving loop that must not call cudaMalloc (which can
 * synchronise the device and take allocator locks).
 *   Arguments, layout, result and return codes: as intattn_decode.
 *   Limit: intattn_decode_workspace_size(B, H, Lk, d) must not exceed
 *   INTATTN_STATIC_SCRATCH_BYTES, else INTATTN_ERR_WORKSPACE (nothing runs).
 *   The array (one per GPU that loads the library, kept until exit) is
 *   shared by every call and keeps the previous call's contents; the kernels
 *   overwrite what they read and clear their own counters, so no clearing is
 *   needed, but two calls on one device that overlap on the GPU (for
 *   example on two streams) race on it: order them on one stream.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  Calls no cudaMalloc, cudaFree or allocating
 *   library routine. */
int intattn_decode_static_scratch(const int8_t *q, const int8_t *k_cache, const int8_t *v_cache,
                                  const intattn_scales_t *scales, int B, int H, int Lk, int Lmax, int d,
                                  float clip_c, int8_t *out, intattn_stream_t stream);

/* Diagnostic for the failure detection: launches one CTA whose wait on a
 * barrier can never complete.  The wait gives up after the kernels' time
 * limit (2 s) and sets the device error word, so a following
 * intattn_device_error(stream) returns INTATTN_ERR_TIMEOUT.  Nothing faults
 * or hangs and the context stays usable. */
int intattn_selftest_timeout(intattn_stream_t stream);

/* Synchronises `stream`, then returns and clears the device error word that a
 * kernel sets when one of its bounded waits runs out (INTATTN_ERR_TIMEOUT) or
 * when parameters derived on the device are out of range
 * (INTATTN_ERR_PARAM_RANGE, see intattn_forward_fp), or INTATTN_OK.
 * INTATTN_ERR_CUDA if the synchronisation itself fails. */
int intattn_device_error(intattn_stream_t stream);

/* Static description of a return code. */
const char *intattn_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* INTATTN_H */
