/*
 * fp8moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts FP8
 * blockwise (W8A8) prefill library, libfp8moe.so.
 *
 * The path, in the order the library runs it:
 *   moe_route        top-k routing with normalised weights, then a stable
 *                    permutation of (token, slot) pairs by expert;
 *   moe_quant_act    BF16 rows -> E4M3 codes with one FP32 scale per
 *                    1x128 group;
 *   moe_route_quant  the two above in one call (fused first launch);
 *   moe_grouped_ffn  grouped gate/up GEMM, unclamped SiLU(gate)*up,
 *                    requantisation of the intermediate, grouped down GEMM
 *                    whose epilogue writes routing-weighted FP32 slot rows;
 *   moe_combine      slot rows summed in slot order, times routed_scaling.
 *
 * Sources (web pages, cited by title and section):
 *   "Full GLM-5.3 streamed FP8 GPU prefill on AVX2 / 2x32GiB SM120",
 *     section "Design": GPU W8A8 routed experts for prefill (>=256 tokens),
 *     unclamped SiLU, expert arithmetic tiled at <=4K rows, explicit
 *     rejection of unsupported dimensions/activation/quantisation, fail
 *     closed.
 *   "Integration for GLM-4.6-FP8 and performance tune on H20", gap table
 *     rows 3, 6, 7: single-wave grid sizing; blockwise FP8 MoE with
 *     zero-padding of a non-128-divisible intermediate (192 -> 256); fused
 *     router chain (gate -> top-k -> dispatch).
 *   "Exact AVX2 FP8 arithmetic conversion avoids costly LUT gathers",
 *     "Semantics and scope": E4M3 format rules; "Real-checkpoint
 *     measurements": top-8 routes with normalised routing weights.
 *   "GLM-5.3-Flash EXL3 on CUDA: a whole prompt pass routes its experts in
 *     one call", "Exactness" and commit text: one call per pass of up to
 *     4,096 rows and more, whole-K accumulation without split-K, row bits
 *     independent of how many rows share the call, routed FP32 rows written
 *     in place, plan -> grouped gate/up -> grouped down -> combine.
 *
 * Conventions for every entry point:
 *   - Every data pointer is DEVICE memory owned by the caller.  The library
 *     allocates nothing, keeps no state between calls and never copies or
 *     repacks weights.  Scratch comes from the caller's workspace, sized by
 *     the *_workspace_bytes queries.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     only enqueue work; they never synchronise and never read device data
 *     back to the host, so a sequence of calls can be captured in a CUDA
 *     graph.
 *   - Arguments are validated on the host before anything is enqueued; a
 *     non-zero moe_status is returned and nothing runs.  There is no CPU
 *     fallback and no silent fallback.
 *   - Faults found on the device (an expert id outside [-1, E) in a
 *     caller-supplied table, a pair index out of range, inconsistent
 *     offsets, a bounded wait that expired) set bits in a status word at the
 *     start of that call's workspace; the affected rows are skipped.
 *     moe_get_device_status reads it.  No kernel traps or spins forever.
 *   - Layouts are row-major.  Alignment: every pointer 16 bytes.
 *   - Requires an sm_100 device (B200); other devices get
 *     MOE_ERR_UNSUPPORTED.
 */
#ifndef FP8MOE_H
#define FP8MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad size, null pointer, out-of-range parameter */
    MOE_ERR_UNSUPPORTED = 2,   /* valid request this library does not implement */
    MOE_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    MOE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than queried */
    MOE_ERR_CUDA = 5,          /* a CUDA runtime/driver call or launch failed */
    MOE_ERR_DEVICE_STATUS = 6  /* moe_get_device_status found device-side faults */
} moe_status;

/* Device status bits (moe_get_device_status). */
#define MOE_DEV_BAD_EXPERT_ID 0x1  /* an id outside [-1, E) in topk_ids */
#define MOE_DEV_BAD_PAIR 0x2       /* a sorted_pairs entry outside [0, T*top_k) */
#define MOE_DEV_BAD_OFFSETS 0x4    /* expert_offsets not monotone or beyond T*top_k */
#define MOE_DEV_WAIT_TIMEOUT 0x8   /* a bounded wait inside a kernel expired */

/* Limits checked on the host. */
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOP_K 32
#define MOE_MAX_INTERMEDIATE 8192
#define MOE_MAX_HIDDEN 16384

/* Human-readable name of a moe_status value (static string). */
MOE_API const char* moe_status_string(int status);

/* ABI version of this header, (major << 16) | minor. */
MOE_API int moe_abi_version(void);

/* Text of the last CUDA failure seen by this thread in a call that returned
 * MOE_ERR_CUDA or MOE_ERR_UNSUPPORTED from the device ("" if none).  The
 * string is owned by the library and valid until the thread's next call. */
MOE_API const char* moe_last_error(void);

/* ---------------------------------------------------------------------------
 * moe_route -- top-k routing and the stable permutation by expert.
 *
 * For each token t, the selectable logits (not NaN, not -Inf) are ordered by
 * value descending, then expert id ascending; the first min(top_k, #selectable)
 * become the token's slots, in that order.  Slot weights are the softmax of
 * the selected logits (FP32, expf), so they sum to 1.  Unfilled slots get
 * id -1 and weight 0.  (Softmax scoring: the tiny workload's statement;
 * top-k with normalised weights: "Exact AVX2 FP8 arithmetic conversion ...",
 * "Real-checkpoint measurements".)
 *
 * The flat pairs p = t*top_k + j with a valid id are then grouped by expert
 * with a stable counting sort: expert_offsets[e] is the exclusive prefix of
 * the per-expert counts (expert_offsets[E] = number of valid pairs, P), and
 * pair p sits at sorted_pairs[expert_offsets[e] + #{p' < p : id(p') = e}].
 * Positions P .. T*top_k-1 of sorted_pairs hold -1.  All integer outputs are
 * deterministic and independent of launch shape.
 *
 *   logits          [T, E]      FP32, read
 *   topk_ids        [T, top_k]  int32, written
 *   topk_w          [T, top_k]  FP32, written
 *   expert_offsets  [E + 1]     int32, written
 *   sorted_pairs    [T * top_k] int32, written
 *   ws, ws_bytes    scratch of at least moe_route_workspace_bytes(T, E, top_k)
 *
 * Limits: T >= 0 (0 is a no-op that still writes expert_offsets = 0),
 * 1 <= E <= 1024, 0 <= top_k <= min(E, 32).
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_route_workspace_bytes(int64_t T, int E, int top_k);
MOE_API int moe_route(const float* logits, int64_t T, int E, int top_k,
              int32_t* topk_ids, float* topk_w,
              int32_t* expert_offsets, int32_t* sorted_pairs,
              void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route_quant -- moe_route and moe_quant_act in one call, the activation
 * quantiser riding in the router's first launch (both read only their own
 * inputs, so neither waits for the other).  This is the fused router chain
 * of "Integration for GLM-4.6-FP8 and performance tune on H20" (gap table
 * row 7: the chain of small router kernels launched as one).
 *
 *   logits, topk_ids, topk_w, expert_offsets, sorted_pairs, ws, ws_bytes:
 *       as for moe_route (the workspace is moe_route_workspace_bytes(T, E,
 *       top_k)); E, top_k: as for moe_route;
 *   x, H, codes, scales: as for moe_quant_act (x [T, H] BF16 bits read;
 *       codes [T, H] uint8 and scales [T, H/128] FP32 written).
 *
 * Results are bit-identical to the two separate calls.  Errors: the union of
 * both calls' argument checks, before anything is enqueued; then as
 * moe_route.  Three kernel launches in total (moe_route alone takes three,
 * moe_quant_act one).
 * ------------------------------------------------------------------------- */
MOE_API int moe_route_quant(const float* logits, const uint16_t* x, int64_t T, int H, int E, int top_k,
                            int32_t* topk_ids, float* topk_w, int32_t* expert_offsets, int32_t* sorted_pairs,
                            uint8_t* codes, float* scales, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route_noalloc -- moe_route without a workspace argument.  The pages
 * have no counterpart: this entry point exists for callers that cannot
 * allocate device memory at all (for example code running inside another
 * runtime's execution hook, which owns and pre-plans every device byte, or
 * a latency-critical path that cannot afford the implicit synchronisation of
 * cudaMalloc).  It allocates nothing; the router's scratch (an arrival
 * counter, block histograms and per-pair ranks) lives in one static device
 * array of 1 MiB + 4 KiB that every GPU loading the library holds until the
 * process exits.
 *   - Same arguments, results and limits as moe_route, and additionally the
 *     scratch of (T, E, top_k) must fit the array: 256 + ceil(T/128)*E*4 +
 *     T*top_k*4 bytes plus alignment (T = 16384, E = 1024, top_k = 8 fits).
 *     Larger requests return MOE_ERR_WORKSPACE before anything is enqueued;
 *     moe_route_noalloc_error() then names the sizes.
 *   - The first call in a CUDA context looks up the array's device address
 *     (cudaGetSymbolAddress) with that context current, and caches it with
 *     the context's id; a later call from another context (for instance
 *     after cudaDeviceReset created a new one) looks it up again.  Make the
 *     first call in a context before any stream capture in it.
 *   - T is capped as for moe_route (MOE_ERR_UNSUPPORTED beyond it).
 *   - All calls share the one array: calls whose kernels overlap on the GPU
 *     (other streams, other host threads) race with each other.  Serialise
 *     them, e.g. on one stream.
 * ------------------------------------------------------------------------- */
MOE_API int moe_route_noalloc(const float* logits, int64_t T, int E, int top_k,
                              int32_t* topk_ids, float* topk_w,
                              int32_t* expert_offsets, int32_t* sorted_pairs, void* stream);
/* Text describing the last rejection or failure of moe_route_noalloc on this
 * thread ("" if none). */
MOE_API const char* moe_route_noalloc_error(void);

/* ---------------------------------------------------------------------------
 * moe_quant_act -- BF16 activations to E4M3 codes with 1x128 group scales.
 *
 * For each token and each group of 128 consecutive columns:
 *   amax = max |x|;  s = amax / 448 (IEEE FP32 divide);  s == 0 -> s = 1;
 *   code = E4M3(x / s), round to nearest even, saturating at +-448
 *   (cvt.rn.satfinite); a group holding NaN or Inf gets s = NaN and every
 *   code 0x7F.  No flush of subnormals on either side of the divide.
 * The rule is the plainest reading of W8A8 with per-token 1x128 activation
 * scales; the pages fix only that activations are FP8 with blockwise scales
 * ("Integration for GLM-4.6-FP8 ...", row 6; "Full GLM-5.3 ...", "Design").
 *
 *   x       [T, H]      BF16 (passed as raw 16-bit words), read
 *   codes   [T, H]      uint8 E4M3, written
 *   scales  [T, H/128]  FP32, written
 *
 * Limits: T >= 0, H % 128 == 0, 128 <= H <= 16384.
 * ------------------------------------------------------------------------- */
MOE_API int moe_quant_act(const uint16_t* x, int64_t T, int H,
                  uint8_t* codes, float* scales, void* stream);

/* ---------------------------------------------------------------------------
 * moe_quant_act_mx -- BF16 activations to MXFP8: E4M3 codes with one UE8M0
 * (power-of-two) scale byte per 32 consecutive values.  The pages name an
 * MXFP8 MoE runtime only as not yet qualified ("Exact AVX2 FP8 arithmetic
 * conversion avoids costly LUT gathers", "Real-checkpoint measurements",
 * caveats); the rule follows the OCP Microscaling Formats:
 *   amax = max |x| over the block; se = floor(log2(amax)) - 8 (8: the
 *   exponent of E4M3's largest value, 448 = 1.75 * 2^8), clamped to
 *   [-127, 127], -127 for amax = 0; scale byte = se + 127 (value 2^se);
 *   code = E4M3(x / 2^se), round to nearest even, saturating at +-448; a
 *   block holding NaN or Inf gets scale byte 0xFF and every code 0x7F.
 *
 *   x       [T, H]     BF16 (raw 16-bit words), read
 *   codes   [T, H]     uint8 E4M3, written
 *   scales  [T, H/32]  uint8 UE8M0, written
 *
 * Limits: T >= 0, H % 32 == 0, 32 <= H <= 16384.
 * ------------------------------------------------------------------------- */
MOE_API int moe_quant_act_mx(const uint16_t* x, int64_t T, int H, uint8_t* codes, uint8_t* scales, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn -- the experts: grouped gate/up GEMM -> SiLU*up ->
 * requantise -> grouped down GEMM -> routing-weighted slot rows.
 *
 * For every valid pair r (token t, slot j, expert e) taken from
 * sorted_pairs / expert_offsets:
 *   g[n] = sum_kb sa[t,kb] * sg[e,n/128,kb] * sum_{k in kb} dec(q[t,k]) dec(Wg[e,n,k])
 *   u[n] likewise with Wu, su;                         (FP32 accumulation)
 *   h[n] = g[n] / (1 + exp(-g[n])) * u[n]              (unclamped SiLU)
 *   (hq, sh) = the moe_quant_act rule applied to h per 128-column group of
 *              the intermediate (columns I..Ip-1 are zero, Ip = ceil(I/128)*128)
 *   o[c] = sum_ib sh[ib] * sd[e,c/128,ib] * sum_{i in ib} dec(hq[i]) dec(Wd[e,c,i])
 *   y[t, j, c] = topk_w[t, j] * o[c]
 * Rows of y for slots with id -1 are not written.  Each row's bits depend
 * only on that row's inputs and the expert's weights: no split-K, fixed
 * K order, tile shapes independent of T ("GLM-5.3-Flash EXL3 on CUDA ...",
 * "Exactness").  Weights are read in place; a non-128-divisible I is padded
 * by out-of-bounds zero fill, not by copies ("Integration for GLM-4.6-FP8
 * ...", row 6).  One call covers all T rows, so each weight tile is streamed
 * from HBM once per call however large T is ("Full GLM-5.3 ...", "Design":
 * <=4K-row tiles without repeating the weight transfer).
 *
 *   codes, act_scales      [T, H] uint8, [T, H/128] FP32  (moe_quant_act output)
 *   topk_ids, topk_w       [T, top_k] int32 / FP32        (moe_route output)
 *   expert_offsets         [E + 1] int32                  (moe_route output)
 *   sorted_pairs           [T * top_k] int32              (moe_route output)
 *   w_gate, w_up           [E, I, H] uint8 E4M3 (K-major: each output row contiguous)
 *   s_gate, s_up           [E, ceil(I/128), H/128] FP32
 *   w_down                 [E, H, I] uint8 E4M3
 *   s_down                 [E, H/128, ceil(I/128)] FP32
 *   y                      [T, top_k, H] FP32, written (valid slots only)
 *   ws, ws_bytes           scratch of at least moe_ffn_workspace_bytes(T, H, I, E, top_k)
 *   stage_events           NULL, or 4 cudaEvent_t handles for profiling: event i
 *                          is recorded on `stream` before stage i (0 = gather of
 *                          the A rows, 1 = gate/up GEMM, 2 = down GEMM) and event
 *                          3 after the down GEMM.  Owned by the caller.
 *
 * Limits: H % 128 == 0, 128 <= H <= 16384; I % 16 == 0, 16 <= I <= 8192;
 * 1 <= E <= 1024; 1 <= top_k <= min(E, 32); T >= 0.  Weight and scale
 * bytes 0x7F/0xFF (E4M3 NaN) are outside the contract.
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_ffn_workspace_bytes(int64_t T, int H, int I, int E, int top_k);
MOE_API int moe_grouped_ffn(const uint8_t* codes, const float* act_scales, int64_t T, int H,
                    const int32_t* topk_ids, const float* topk_w, int top_k,
                    const int32_t* expert_offsets, const int32_t* sorted_pairs,
                    int E, int I,
                    const uint8_t* w_gate, const float* s_gate,
                    const uint8_t* w_up, const float* s_up,
                    const uint8_t* w_down, const float* s_down,
                    float* y, void* ws, size_t ws_bytes, void* stream,
                    void* const* stage_events);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn_mx -- the experts of the MXFP8 variant: the same routing
 * inputs, steps and y output as moe_grouped_ffn, with every operand in the
 * OCP MX format (E4M3 codes, one UE8M0 scale byte per 32 values along K)
 * and the scales applied by the tensor core inside each K = 32 step.  The
 * pages list an MXFP8 MoE runtime only as not yet qualified ("Exact AVX2 FP8
 * arithmetic conversion avoids costly LUT gathers", "Real-checkpoint
 * measurements", caveats); the arithmetic follows the OCP Microscaling
 * Formats.  For every valid pair (token t, slot j, expert e):
 *   g[n] = sum_k 2^(sa[t,k/32]-127) dec(q[t,k]) 2^(sg[e,n,k/32]-127) dec(Wg[e,n,k])
 *   u[n] likewise with Wu, su;                         (FP32 accumulation)
 *   h[n] = g[n] / (1 + exp(-g[n])) * u[n]              (unclamped SiLU)
 *   (hq, sh) = the moe_quant_act_mx rule applied to h per 32 columns
 *   o[c] = sum_i 2^(sh[i/32]-127) dec(hq[i]) 2^(sd[e,c,i/32]-127) dec(Wd[e,c,i])
 *   y[t, j, c] = topk_w[t, j] * o[c]
 * Rows of y for slots with id -1 are not written; each row's bits depend
 * only on that row's inputs and the expert's weights.  Follow with
 * moe_combine.
 *
 *   codes, act_scales      [T, H] uint8, [T, H/32] uint8  (moe_quant_act_mx output)
 *   topk_ids, topk_w, expert_offsets, sorted_pairs   as moe_grouped_ffn
 *   w_gate, w_up           [E, I, H] uint8 E4M3
 *   s_gate, s_up           UE8M0 bytes of [E, I, H/32], packed by moe_mx_pack_scales
 *   w_down                 [E, H, I] uint8 E4M3
 *   s_down                 UE8M0 bytes of [E, H, I/32], packed by moe_mx_pack_scales
 *   y                      [T, top_k, H] FP32, written (valid slots only)
 *   ws, ws_bytes           scratch of at least moe_ffn_mx_workspace_bytes(T, H, I, E, top_k)
 *   stage_events           as moe_grouped_ffn
 *
 * Limits: H % 128 == 0, 128 <= H <= 16384; I % 32 == 0, 128 <= I <= 8192;
 * 1 <= E <= 1024; 1 <= top_k <= min(E, 32); T >= 0.  Scale bytes 0xFF (NaN)
 * and code bytes 0x7F/0xFF in the weights are outside the contract.
 * Errors as moe_grouped_ffn.
 * ------------------------------------------------------------------------- */
/* moe_mx_pack_scales -- weight scale bytes from the checkpoint layout
 * src [E, R, K/32] (row r's scale of columns 32c..32c+31 at byte c) into the
 * layout the MX FFN reads: dst [E][G][R][16], G = ceil(K/512), where byte
 * (e, g, r, b) holds chunk 16g + b of row r (127, i.e. 2^0, for chunks at or
 * past K/32).  Each 16-byte word covers four K blocks of one row, and 32
 * consecutive rows' words are contiguous: the kernel loads a tile's scales
 * for four K blocks with one coalesced request per lane.  A one-time
 * transformation of static weights (no counterpart on the pages).
 *   src  device, read;  dst device, moe_mx_packed_scales_bytes(E, R, K) bytes, written
 * Limits: E >= 0, R >= 1, K % 32 == 0, K >= 32.  Errors: MOE_ERR_INVALID_ARG,
 * MOE_ERR_ALIGNMENT (dst not 16-byte aligned), MOE_ERR_CUDA. */
MOE_API size_t moe_mx_packed_scales_bytes(int64_t E, int R, int K);
MOE_API int moe_mx_pack_scales(const uint8_t* src, int64_t E, int R, int K, uint8_t* dst, void* stream);
MOE_API size_t moe_ffn_mx_workspace_bytes(int64_t T, int H, int I, int E, int top_k);
MOE_API int moe_grouped_ffn_mx(const uint8_t* codes, const uint8_t* act_scales, int64_t T, int H,
                               const int32_t* topk_ids, const float* topk_w, int top_k,
                               const int32_t* expert_offsets, const int32_t* sorted_pairs, int E, int I,
                               const uint8_t* w_gate, const uint8_t* s_gate, const uint8_t* w_up,
                               const uint8_t* s_up, const uint8_t* w_down, const uint8_t* s_down, float* y,
                               void* ws, size_t ws_bytes, void* stream, void* const* stage_events);

/* ---------------------------------------------------------------------------
 * moe_combine -- out[t, :] = routed_scaling * sum_{j : id(t,j) >= 0} y[t, j, :]
 *
 * Summed in FP32 in slot order j = 0 .. top_k-1 (no atomics), then scaled:
 * routed scaling is kept with the routed-expert sum ("Full GLM-5.3 ...",
 * "Design"), and the rows are FP32 ("GLM-5.3-Flash EXL3 on CUDA ...",
 * commit text).  A token with no valid slot gets exact zeros.  out_bf16,
 * when not NULL, receives the round-to-nearest-even BF16 of out_f32.
 *
 *   y          [T, top_k, H] FP32, read (rows of valid slots)
 *   topk_ids   [T, top_k] int32, read
 *   out_f32    [T, H] FP32, written
 *   out_bf16   [T, H] BF16 words, written, nullable
 *   ws, ws_bytes  at least moe_combine_workspace_bytes() (status word)
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_combine_workspace_bytes(void);
MOE_API int moe_combine(const float* y, const int32_t* topk_ids, int64_t T, int H, int top_k, int E,
                float routed_scaling, float* out_f32, uint16_t* out_bf16,
                void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn_combine -- moe_grouped_ffn with moe_combine fused into the
 * down GEMM's epilogue, so the routed FP32 rows are summed where they are
 * written ("GLM-5.3-Flash EXL3 on CUDA ...", commit text: routed FP32 rows
 * written in place, plan -> grouped gate/up -> grouped down -> combine).
 * Arguments as
 * moe_grouped_ffn (y is still written: it carries the slot rows between the
 * GEMM's tiles) plus routed_scaling, out_f32 [T, H] and out_bf16 (nullable) as
 * moe_combine.  The down items run n-tile-major, so a token's k slot rows of
 * one 256-column block are produced close together.  Each slot row segment
 * counts an arrival per (token, n-tile, column half); the arrival that
 * completes a token's valid slots makes its warp sum the token's slot rows in
 * slot order.  The arithmetic is moe_combine's (from zero, valid slots in
 * order, times routed_scaling), so the result equals moe_grouped_ffn followed
 * by moe_combine bit for bit, whatever the order of arrival.  Rows of tokens
 * without a valid slot are written as zeros.  Workspace:
 * moe_ffn_workspace_bytes (it includes the arrival counters).
 * ------------------------------------------------------------------------- */
MOE_API int moe_grouped_ffn_combine(const uint8_t* codes, const float* act_scales, int64_t T, int H,
                                    const int32_t* topk_ids, const float* topk_w, int top_k,
                                    const int32_t* expert_offsets, const int32_t* sorted_pairs, int E, int I,
                                    const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up,
                                    const float* s_up, const uint8_t* w_down, const float* s_down, float* y,
                                    float routed_scaling, float* out_f32, uint16_t* out_bf16, void* ws,
                                    size_t ws_bytes, void* stream, void* const* stage_events);

/* ---------------------------------------------------------------------------
 * Shared-expert slot.  The pages plan a shared expert as one more slot after
 * the routed ones ("GLM-5.3-Flash EXL3 on CUDA ...": all nine slots planned
 * with E+1 expert ids, the shared id skipped before any routed payload is
 * read, routed FP32 rows written in place).  Readings: the shared slot is
 * slot top_k, id E, weight 1; the caller computes the shared expert and
 * writes its row into that slot of y; the combine adds it after the routed
 * scaling, out = routed_scaling * sum(routed slots) + shared (the pages keep
 * routed scaling and the shared experts as separate parts of the layer).
 *
 * moe_route_shared: moe_route whose topk_ids / topk_w are [T, top_k+1] with
 *   slot top_k = (E, 1.0) and whose sorted_pairs is [T*(top_k+1)]; the
 *   permutation holds the routed pairs only (the shared id is skipped), so
 *   moe_grouped_ffn with top_k+1 slots computes the routed rows and leaves the
 *   shared slot's rows of y untouched.  Workspace:
 *   moe_route_workspace_bytes(T, E, top_k+1).  1 <= top_k <= 31.
 * moe_combine_shared: moe_combine over top_k slots (the shared one
 *   included) in which the slots holding id E are summed apart (slot order)
 *   and added to routed_scaling * (sum of the routed slots).
 * ------------------------------------------------------------------------- */
MOE_API int moe_route_shared(const float* logits, int64_t T, int E, int top_k, int32_t* topk_ids, float* topk_w,
                             int32_t* expert_offsets, int32_t* sorted_pairs, void* ws, size_t ws_bytes,
                             void* stream);
MOE_API int moe_combine_shared(const float* y, const int32_t* topk_ids, int64_t T, int H, int top_k, int E,
                               float routed_scaling, float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes,
                               void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism across `world` GPUs.  The pages describe only
 * single-GPU and tensor-parallel layers; the reading taken here is that
 * the layer shards by expert with one exchange on each side, and each
 * token's k slot rows are summed on its home GPU in slot order, so a row's
 * bits do not depend on the sharding -- "GLM-5.3-Flash EXL3 on CUDA ...",
 * exactness note).  Rank r owns experts [r*E/world, (r+1)*E/world) and is
 * home to tokens [r*T_home, (r+1)*T_home).  Every rank routes all T tokens.
 *
 * moe_ep_plan: from the replicated topk_ids [T, top_k] (read):
 *   local_ids  [T, top_k] int32: the rank's own experts renumbered from 0,
 *              -1 for the others (input of moe_permute / the grouped FFN);
 *   send_rows  [T*top_k]  int32: row of each own pair in the rank's send
 *              buffer (-1: not own), grouped by home rank, pair order inside
 *              each group (y_rows of moe_grouped_ffn_rows);
 *   recv_rows  [T_home, top_k] int32: row of each home slot in the receive
 *              buffer, grouped by owner rank in rank order (-1: empty slot;
 *              moe_combine_rows);
 *   offs_oh, offs_ho  [world*world + 1] int32: exclusive prefixes of the
 *              pair counts by (owner, home) and by (home, owner); rank r
 *              sends offs_oh[r*w+h+1] - offs_oh[r*w+h] rows to home h and
 *              receives offs_ho[r*w+o+1] - offs_ho[r*w+o] rows from owner o.
 * Both sides take rows in pair order, so no indices travel with them.
 * Limits: E % world == 0, world*world <= 1024, T_home*world >= T; workspace
 * moe_ep_plan_workspace_bytes(T, top_k, world).
 *
 * moe_permute: the stable permutation of moe_route (A2) on caller-given ids
 * (ids outside [0, E) are skipped); workspace moe_route_workspace_bytes.
 *
 * moe_grouped_ffn_rows: moe_grouped_ffn whose down epilogue writes pair p
 * to row y_rows[p] of y (y_nrows rows; -1: not written; a row >= y_nrows is
 * a device fault, MOE_DEV_BAD_PAIR).  y_rows == NULL is moe_grouped_ffn.
 *
 * moe_combine_rows: out[t] = routed_scaling * sum over j in slot order of
 * y[rows[t*top_k + j]] for rows >= 0 (rows >= y_nrows: MOE_DEV_BAD_PAIR);
 * ws as moe_combine.
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_ep_plan_workspace_bytes(int64_t T, int top_k, int world);
MOE_API int moe_ep_plan(const int32_t* topk_ids, int64_t T, int top_k, int E, int world, int rank, int64_t T_home,
                        int32_t* local_ids, int32_t* send_rows, int32_t* recv_rows, int32_t* offs_oh,
                        int32_t* offs_ho, void* ws, size_t ws_bytes, void* stream);
MOE_API int moe_permute(const int32_t* ids, int64_t T, int E, int top_k, int32_t* expert_offsets,
                        int32_t* sorted_pairs, void* ws, size_t ws_bytes, void* stream);
MOE_API int moe_grouped_ffn_rows(const uint8_t* codes, const float* act_scales, int64_t T, int H,
                                 const int32_t* topk_ids, const float* topk_w, int top_k,
                                 const int32_t* expert_offsets, const int32_t* sorted_pairs, int E, int I,
                                 const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up, const float* s_up,
                                 const uint8_t* w_down, const float* s_down, float* y, const int32_t* y_rows,
                                 int64_t y_nrows, void* ws, size_t ws_bytes, void* stream,
                                 void* const* stage_events);
MOE_API int moe_combine_rows(const float* y, int64_t y_nrows, const int32_t* rows, int64_t T, int H, int top_k,
                             float routed_scaling, float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes,
                             void* stream);

/* ---------------------------------------------------------------------------
 * moe_layer -- the whole routed-expert layer in one call: moe_route_quant,
 * moe_grouped_ffn and moe_combine, stream-ordered, over one caller
 * workspace that also holds the intermediates (codes, scales, routing,
 * permutation, slot rows y).  Results are those of the three calls.
 *
 *   logits [T, E] FP32, x [T, H] BF16 bits: read;
 *   w_* / s_*: as for moe_grouped_ffn; routed_scaling, out_f32 [T, H],
 *   out_bf16 (nullable): as for moe_combine;
 *   ws, ws_bytes: at least moe_layer_workspace_bytes(T, H, I, E, top_k).
 *
 * Errors: as the three calls (the first failing one's status is returned;
 * the calls before it stay enqueued).  Limits: the three calls' limits, and
 * top_k >= 1.
 *
 * moe_layer_plan_create captures the same sequence for fixed pointers and
 * sizes into a CUDA graph (thread-local stream capture on a private stream;
 * nothing runs at creation) and instantiates it.  moe_layer_plan_launch
 * enqueues the graph on `stream`: one launch per layer instead of seven
 * kernel launches, three status memsets and the host-side checks.  The
 * plan reads its inputs from, and writes its outputs to, the addresses given
 * at creation, so a caller copies each batch into them.  stage_events
 * (nullable) are 6 cudaEvent_t recorded inside the graph at the start,
 * before the gather, gate/up and down launches, after the down launch, and
 * at the end.  A plan belongs to the device current at creation; destroy it
 * before its buffers.  One plan's launches must not overlap each other.
 * The pages' counterpart: the router chain and the layer captured in-graph
 * ("Integration for GLM-4.6-FP8 and performance tune on H20", gap table
 * row 7).
 *
 * moe_layer_get_device_status: synchronous; ORs the status words of the
 * three calls held in a layer workspace (moe_get_device_status semantics).
 * ------------------------------------------------------------------------- */
typedef struct moe_layer_plan moe_layer_plan;
MOE_API size_t moe_layer_workspace_bytes(int64_t T, int H, int I, int E, int top_k);
MOE_API int moe_layer(const float* logits, const uint16_t* x, int64_t T, int H, int E, int top_k, int I,
                      const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up, const float* s_up,
                      const uint8_t* w_down, const float* s_down, float routed_scaling,
                      float* out_f32, uint16_t* out_bf16, void* ws, size_t ws_bytes, void* stream);
MOE_API int moe_layer_plan_create(moe_layer_plan** plan, const float* logits, const uint16_t* x, int64_t T,
                                  int H, int E, int top_k, int I, const uint8_t* w_gate, const float* s_gate,
                                  const uint8_t* w_up, const float* s_up, const uint8_t* w_down,
                                  const float* s_down, float routed_scaling, float* out_f32, uint16_t* out_bf16,
                                  void* ws, size_t ws_bytes, void* const* stage_events);
/* moe_layer_plan_create with options: flags = MOE_LAYER_FUSED_COMBINE uses
 * moe_grouped_ffn_combine in place of moe_grouped_ffn + moe_combine (the
 * stage events then mark the start, the gather, gate/up and down launches,
 * the end of the fused down launch, and the end). */
#define MOE_LAYER_FUSED_COMBINE 1
MOE_API int moe_layer_plan_create_ex(moe_layer_plan** plan, const float* logits, const uint16_t* x, int64_t T,
                                     int H, int E, int top_k, int I, const uint8_t* w_gate, const float* s_gate,
                                     const uint8_t* w_up, const float* s_up, const uint8_t* w_down,
                                     const float* s_down, float routed_scaling, float* out_f32, uint16_t* out_bf16,
                                     void* ws, size_t ws_bytes, void* const* stage_events, int flags);
MOE_API int moe_layer_plan_launch(moe_layer_plan* plan, void* stream);
MOE_API void moe_layer_plan_destroy(moe_layer_plan* plan);
MOE_API int moe_layer_get_device_status(const void* ws, int64_t T, int H, int I, int E, int top_k,
                                        int* status_out);

/* ---------------------------------------------------------------------------
 * moe_get_device_status -- synchronously read the
 * status word at the start of a workspace used by moe_route,
 * moe_grouped_ffn or moe_combine.  Waits for all work on the device.
 * *status_out receives the OR of the MOE_DEV_* bits seen since the last
 * call on that workspace started; returns MOE_OK, or MOE_ERR_CUDA.
 * ------------------------------------------------------------------------- */
MOE_API int moe_get_device_status(const void* ws, int* status_out);

/* ---------------------------------------------------------------------------
 * Test hooks (no counterpart on the pages).
 *   moe_debug_encode: in[n] FP32 -> out[n] uint8 E4M3, the encoder the
 *   kernels use (cvt.rn.satfinite.e4m3x2).
 * ------------------------------------------------------------------------- */
MOE_API int moe_debug_encode(const float* in, int64_t n, uint8_t* out, void* stream);

/* moe_ffn_intermediate: device pointers into a workspace last used by
 * moe_grouped_ffn with the same (T, H, I, top_k): the requantised
 * intermediate codes [T*top_k, Ip] and their scales [T*top_k, ceil(I/128)],
 * rows in expert order (row r belongs to pair sorted_pairs[r]).  Host
 * arithmetic only; nothing is read from the device. */
MOE_API int moe_ffn_intermediate(const void* ws, int64_t T, int H, int I, int top_k,
                                 const uint8_t** h_codes, const float** h_scales);

/* moe_debug_grouped_down: the down GEMM of moe_grouped_ffn alone, on an
 * intermediate the caller supplies: h_codes [T*top_k, Ip] uint8 E4M3 and
 * h_scales [T*top_k, ceil(I/128)] FP32, rows in expert order (row r belongs
 * to pair sorted_pairs[r]; rows at and beyond expert_offsets[E] are not
 * read).  Writes y [T, top_k, H] FP32 for the valid pairs exactly as
 * moe_grouped_ffn's down stage does (same kernel, same tiles).  It lets a
 * test feed one and the same intermediate to this path and to an
 * independent implementation, and so check the down projection and the
 * combine without the requantisation decisions of the gate/up stage.
 * Workspace: at least moe_combine_workspace_bytes() (the status word).
 * Limits and errors as moe_grouped_ffn. */
MOE_API int moe_debug_grouped_down(const uint8_t* h_codes, const float* h_scales, int64_t T, int H, int top_k,
                                   const float* topk_w, const int32_t* expert_offsets, const int32_t* sorted_pairs,
                                   int E, int I, const uint8_t* w_down, const float* s_down, float* y, void* ws,
                                   size_t ws_bytes, void* stream);

/* moe_ffn_mx_intermediate: device pointers into a workspace last used by
 * moe_grouped_ffn_mx with the same (T, H, I, top_k): the MX intermediate
 * codes [T*top_k, Ip] (columns I..Ip-1 unspecified, Ip = ceil(I/128)*128)
 * and scale bytes [G][T*top_k][16], G = ceil(Ip/512): the scale of row r,
 * columns 32c..32c+31 is byte (c/16 * T*top_k + r) * 16 + c%16 (chunks c >=
 * I/32 unspecified); rows in expert order.  Host arithmetic only. */
MOE_API int moe_ffn_mx_intermediate(const void* ws, int64_t T, int H, int I, int top_k,
                                    const uint8_t** h_codes, const uint8_t** h_scales);

/* moe_debug_grouped_down_mx: the down GEMM of moe_grouped_ffn_mx alone, on
 * an intermediate the caller supplies in the layout moe_ffn_mx_intermediate
 * describes (h_codes [T*top_k, Ip], h_scales [G][T*top_k][16], expert
 * order; scale bytes of chunks at or past I/32 are not used), with s_down
 * packed by moe_mx_pack_scales.  Writes y as moe_grouped_ffn_mx's down stage does (same kernel).
 * Workspace: at least moe_combine_workspace_bytes().  Limits and errors as
 * moe_grouped_ffn_mx. */
MOE_API int moe_debug_grouped_down_mx(const uint8_t* h_codes, const uint8_t* h_scales, int64_t T, int H,
                                      int top_k, const float* topk_w, const int32_t* expert_offsets,
                                      const int32_t* sorted_pairs, int E, int I, const uint8_t* w_down,
                                      const uint8_t* s_down, float* y, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8MOE_H */
