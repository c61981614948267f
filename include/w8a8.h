/*
 * w8a8.h - C ABI of libw8a8, the W8A8 INT8 MoE expert-FFN forward for NVIDIA B200 (sm_100a).
 *
 * Method (sources are the pages' titles and sections):
 *   - "Qwen3-30B-A3B-Instruct-2507-quantized.w8a8" explainer, section 二: weights int8 per
 *     output channel, symmetric min-max, static; activations int8 per token, dynamic.
 *     Section 三 3.1: mlp.gate maps the hidden state to one score per expert, softmax, top-8;
 *     the gate is never quantized (ignore list entry re:.*mlp.gate$).
 *   - "Qwen3.6-35B-A3B-w8a8量化配置深度解读：config.json与recipe.yaml关键参数解析",
 *     block config_groups.group_0: the same scheme as explicit fields.
 *   - "Qwen3-1.7B-W4A8-V1" explainer, section "4bit 权重": int4 two's-complement packed
 *     weights with one scale per group of 128 along K; section "8bit 激活": dynamic
 *     per-token int8 activations.
 *   - "Qwen3-235B-A22B-quantized.w8a8" explainer, model table and shard contents: 128
 *     experts, 8 per token, gate_proj/up_proj/down_proj in INT8, mlp.gate in bf16.
 *   - "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战", section 二 2.2:
 *     gate_proj and up_proj of an expert concatenated along the output dimension into
 *     gate_up_proj; down_proj kept separate.
 *
 * Each declaration below names the passage that defines its operation. Conventions for every
 * entry point:
 *   - Pointers are device memory owned by the caller unless stated otherwise; the library
 *     never allocates, frees or retains them. bf16 tensors are passed as their raw 16-bit
 *     patterns (w8a8_bf16). All tensors are row-major and contiguous.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) on the current CUDA device. Calls on different streams are safe when each uses
 *     its own outputs and workspace.
 *   - The return value is a status code (W8A8_OK or a negative W8A8_ERR_*). Argument and
 *     shape checks happen on the host before anything is enqueued; a rejected call enqueues
 *     nothing. Faults found on the device (a wait that ran out, an out-of-range expert id)
 *     set a device error word that w8a8_check_status() reports.
 *   - Shape rules: hidden sizes and reduction lengths are multiples of 128 (the TMA/MMA
 *     K-block), the expert intermediate size I a multiple of 128, E <= 256, 1 <= k <= 16.
 */
#ifndef W8A8_H_
#define W8A8_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t w8a8_bf16; /* raw bfloat16 bits */
typedef void* w8a8_stream;  /* cudaStream_t */

#define W8A8_OK 0
#define W8A8_ERR_ARG (-1)         /* null pointer, negative or inconsistent size */
#define W8A8_ERR_UNSUPPORTED (-2) /* shape or alignment outside the supported set */
#define W8A8_ERR_WORKSPACE (-3)   /* workspace smaller than the size query returned */
#define W8A8_ERR_LAUNCH (-4)      /* a CUDA call or kernel launch failed */
#define W8A8_ERR_DEVICE (-5)      /* the device error word was set (see w8a8_check_status) */

#define W8A8_W_INT8_PER_CHANNEL 0 /* w: int8 [N, K], sw: fp32 [N] */
#define W8A8_W_INT4_PER_GROUP 1   /* w: uint8 [N, K/2] packed int4, sw: fp32 [N, K/group] */

/* Library version, major * 10000 + minor * 100 + patch. */
int w8a8_version(void);

/* Static English text for a status code. */
const char* w8a8_status_string(int status);

/* Synchronises `stream`, then reads and clears the device error word of the current device.
 * Returns W8A8_ERR_DEVICE if any kernel since the last check reported a fault, W8A8_ERR_LAUNCH
 * if the stream itself reports a CUDA error, else W8A8_OK. */
int w8a8_check_status(w8a8_stream stream);

/* Static per-output-channel int8 weight quantisation (offline weight preparation).
 * Defined by: "Qwen3.6-35B-A3B-w8a8量化配置深度解读：config.json与recipe.yaml关键参数解析", block
 * config_groups.group_0.weights (num_bits 8, strategy channel, symmetric, dynamic false, min-max
 * observer); "Qwen3-30B-A3B-Instruct-2507-quantized.w8a8" explainer, section 二.
 *   w      bf16 [G, N, K]   G blocks (experts) of nn.Linear weights [out = N, in = K]
 *   q      int8 [G, N, K]   codes clamp(rne(w / scale), -127, 127)
 *   scale  fp32 [G, N]      max |w[g, n, :]| / 127 (0 for an all-zero row)
 * K must be a multiple of 8. */
int w8a8_quantize_weight_per_channel(const w8a8_bf16* w, int64_t G, int64_t N, int64_t K, int8_t* q,
                                     float* scale, w8a8_stream stream);

/* Symmetric int4 weight quantisation with one scale per `group` consecutive K values.
 * Defined by: "Qwen3-1.7B-W4A8-V1" explainer, section "4bit 权重", items 1 (group_size 128) and 2
 * (two's-complement codes packed two per byte).
 *   w       bf16 [N, K]
 *   packed  uint8 [N, K/2]   byte i = code(2i) & 0xF | (code(2i+1) & 0xF) << 4, codes in [-7, 7]
 *   scale   fp32 [N, K/group] max |w| over the group / 7
 * group must be 128 and K a multiple of it. */
int w8a8_quantize_weight_int4_per_group(const w8a8_bf16* w, int64_t N, int64_t K, int group, uint8_t* packed,
                                        float* scale, w8a8_stream stream);

/* Dynamic per-token symmetric int8 activation quantisation.
 * Defined by: the group_0.input_activations block of the Qwen3.6-35B-A3B-w8a8 config page
 * (num_bits 8, strategy token, symmetric, dynamic true); "Qwen3-1.7B-W4A8-V1" explainer,
 * section "8bit 激活" (each token's scale computed online).
 *   x      bf16 [T, K]
 *   q      int8 [T, K]   clamp(rne(x / scale), -127, 127)
 *   scale  fp32 [T]      max |x[t, :]| / 127 (0 for an all-zero token)
 * K must be a multiple of 8. T = 0 is a no-op. */
int w8a8_quant_act_per_token(const w8a8_bf16* x, int64_t T, int64_t K, int8_t* q, float* scale,
                             w8a8_stream stream);

/* Defined by: "Qwen3-30B-A3B-Instruct-2507-quantized.w8a8" explainer, section 三 3.1 (mlp.gate
 * maps the hidden state to one score per expert, softmax, top-8) and the recipe's ignore list
 * (re:.*mlp.gate$: the gate stays bf16); "Qwen3-235B-A22B-quantized.w8a8" model table (128
 * experts, 8 per token).
 * BF16 router (never quantised): logits = x . wg^T (+ bias) accumulated in fp32 on the tensor
 * cores, softmax over the E experts, top-k by descending probability (equal values: lower
 * expert first), weights renormalised over the k selected experts when renorm != 0.
 *   x              bf16 [T, H]
 *   wg             bf16 [E, H]   (nn.Linear layout)
 *   bias           fp32 [E] or NULL (added to the logits; for routing stress tests)
 *   topk_ids       int32 [T, k]  slot j = j-th most probable expert
 *   topk_w         fp32 [T, k]
 *   expert_counts  int32 [E] or NULL: number of tokens routed to each expert
 * H % 128 == 0, 1 <= E <= 256, 1 <= k <= min(16, E). */
int w8a8_moe_route(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, int64_t T, int64_t H, int64_t E,
                   int k, int renorm, int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                   w8a8_stream stream);

/* Byte offsets of the intermediates that w8a8_moe_forward leaves in its workspace (every
 * region 256-byte aligned). Rows are "sorted rows": the T*k assignments grouped by expert,
 * ordered by token inside an expert; A_pad = T*k rounded up to a multiple of 128.
 *   topk_ids int32 [T, k]; topk_w fp32 [T, k]; tile_counts int32 [ceil(T/128), E];
 *   offsets int32 [E+1] (rows of expert e: offsets[e] .. offsets[e+1]-1);
 *   perm int32 [T*k] (sorted row -> assignment t*k + j); sx fp32 [T] (token scales);
 *   sx_sorted fp32 [A_pad]; xq int8 [A_pad, H] (token codes in sorted-row order);
 *   h bf16 [A_pad, I] (SiLU(gate)*up); s_h fp32 [A_pad]; hq int8 [A_pad, I];
 *   o bf16 [T*k, H] (expert outputs in slot order t*k + j);
 *   logits fp32 [T, E] (router logits; written only for short batches, T <= 512);
 *   sync uint32 (grid-barrier counter of the fused short-batch front end, T <= 128). */
typedef struct {
  size_t topk_ids, topk_w, tile_counts, offsets, perm, sx, sx_sorted, xq, h, s_h, hq, o, logits, sync;
  size_t total;
} w8a8_moe_ws_layout;

/* Fills *layout for the given shape. Returns W8A8_ERR_ARG / W8A8_ERR_UNSUPPORTED on bad
 * shapes. */
int w8a8_moe_workspace_layout(int64_t T, int64_t H, int64_t E, int k, int64_t I, w8a8_moe_ws_layout* layout);

/* Workspace bytes w8a8_moe_forward needs for this shape (0 if the shape is rejected). */
size_t w8a8_moe_workspace_size(int64_t T, int64_t H, int64_t E, int k, int64_t I);

/* Defined by: the group_0 block of the Qwen3.6-35B-A3B-w8a8 config page (int8 per-channel
 * static weights, int8 per-token dynamic activations for every expert Linear, gate_proj,
 * up_proj and down_proj alike); "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战",
 * section 二 2.2 (gate_proj and up_proj concatenated into gate_up_proj); the router as above.
 * W8A8 MoE expert-FFN forward of one Qwen3-MoE layer:
 *   route (bf16) -> per-token int8 x -> grouped int8 gate_up GEMM (int32) -> dequant
 *   ((acc * s_x) * s_gu), SiLU(gate) * up -> bf16 h -> per-row int8 requantisation of h ->
 *   grouped int8 down GEMM -> dequant ((acc * s_h) * s_d) -> bf16 o -> y[t] = bf16(sum_j
 *   w[t,j] * o[t,j]) (one fp32 fused multiply-add per slot, in slot order from 0).
 *   x     bf16 [T, H];  wg bf16 [E, H];  bias fp32 [E] or NULL
 *   wgu   int8 [E, 2I, H]  packed gate_up: rows 0..I-1 gate_proj, rows I..2I-1 up_proj
 *   s_gu  fp32 [E, 2I]     per-channel scales of wgu
 *   wd    int8 [E, H, I];  s_d fp32 [E, H]
 *   workspace  device buffer of at least w8a8_moe_workspace_size() bytes, 256-byte aligned;
 *              it keeps the intermediates listed in w8a8_moe_ws_layout after the call.
 *   y     bf16 [T, H]
 * H % 128 == 0, I % 128 == 0, E <= 256, 1 <= k <= min(16, E). T = 0 is a no-op. */
int w8a8_moe_forward(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                     const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H, int64_t E,
                     int k, int64_t I, int renorm, void* workspace, size_t workspace_bytes, w8a8_bf16* y,
                     w8a8_stream stream);

/* ---- Expert parallelism: the forward split at its two exchange points ----------------------
 * Defined by: "Qwen3-235B-A22B-quantized.w8a8" file-structure explainer, the model table (128
 * experts, 8 per token) and the shard index section (the weights are sharded so that several cards
 * load and serve the model together). Read as expert parallelism: rank r of W holds experts
 * [r E/W, (r+1) E/W); each rank routes its own tokens, sends every assignment's int8 row and fp32
 * scale to the rank of its expert, runs the expert FFN on what it receives, and gets the bf16
 * expert outputs back for its ordered combine. Every step is row-wise, so the result equals
 * w8a8_moe_forward on the same tokens bit for bit. The exchanges themselves are the caller's
 * (the package's ep.py uses torch.distributed all-to-all); these entries are the compute between.
 *
 * w8a8_moe_route_group: steps 1 and 2 of w8a8_moe_forward on T local tokens (router, softmax,
 * top-k, grouping by global expert, per-token int8 quantisation into the sorted rows). The
 * workspace has the layout w8a8_moe_workspace_layout(T, H, E, k, 128, .) gives and at least its
 * total; the call fills topk_ids, topk_w, offsets (sorted rows of each global expert; with experts
 * in contiguous blocks per rank, the rows for each destination rank are consecutive), perm, sx,
 * sx_sorted and xq. Shape rules and errors as w8a8_moe_forward. */
int w8a8_moe_route_group(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, int64_t T, int64_t H, int64_t E,
                         int k, int renorm, void* workspace, size_t workspace_bytes, w8a8_stream stream);

/* Workspace bytes of w8a8_moe_experts for A rows and Ew experts (0 if rejected: H or I not a
 * multiple of 128, Ew outside [1, 256]). */
size_t w8a8_moe_experts_workspace_size(int64_t A, int64_t H, int64_t I, int64_t Ew);

/* Steps 3-5 of w8a8_moe_forward on A received rows: grouped gate_up GEMM with dequant and
 * SiLU(gate)*up, per-row requantisation of h, grouped down GEMM with dequant; o [A, H] bf16, row r
 * the output of input row r.
 *   xq int8 [A, H] (16-byte aligned) and sx fp32 [A]: the rows and their per-token scales;
 *   group_offsets_host: HOST array [G+1], offsets[0] = 0, non-decreasing, offsets[G] = A (else
 *   W8A8_ERR_ARG), group g = rows [offsets[g], offsets[g+1]); group g uses expert g % weight_groups
 *   of the Ew experts in wgu [Ew, 2I, H] / s_gu [Ew, 2I] / wd [Ew, H, I] / s_d [Ew, H]
 *   (weight_groups 0: expert g, G <= Ew) -- with W source ranks and E/W local experts, G = W * E/W
 *   groups in source-major order and weight_groups = E/W; G <= 1024;
 *   workspace of w8a8_moe_experts_workspace_size(A, H, I, Ew) bytes (256-byte aligned).
 * The call regroups the rows by expert (a row gather into the workspace, the map built on the
 * host and copied), runs the grouped GEMMs on the experts' row blocks, and the down GEMM writes
 * each output row back at its input position. All device memory except group_offsets_host owned
 * by the caller. */
int w8a8_moe_experts(const int8_t* xq, const float* sx, const int* group_offsets_host, int64_t G,
                     int64_t weight_groups, int64_t A, int64_t H, int64_t I, int64_t Ew, const int8_t* wgu,
                     const float* s_gu, const int8_t* wd, const float* s_d, void* workspace, size_t workspace_bytes,
                     w8a8_bf16* o, w8a8_stream stream);

/* Step 6 of w8a8_moe_forward from expert outputs in sorted-row order: o_sorted [T*k, H] bf16 (row
 * r = sorted row r, as w8a8_moe_route_group ordered them), perm and topk_w from the same call;
 * o_slots [T*k, H] bf16 is scratch (receives the rows in slot order t*k + j); y [T, H] bf16 =
 * bf16(fma chain over j = 0..k-1 of topk_w[t, j] * o[t, j, :]). A perm entry outside [0, T*k) sets
 * the device error word (W8A8_ERR_DEVICE at the next w8a8_check_status) and its row is skipped.
 * H % 128 == 0, k <= 16. */
int w8a8_moe_combine_sorted(const w8a8_bf16* o_sorted, const int* perm, const float* topk_w, int64_t T, int64_t H,
                            int k, w8a8_bf16* o_slots, w8a8_bf16* y, w8a8_stream stream);

/* Workspace of w8a8_moe_forward_shared: the routed layer's regions (as w8a8_moe_ws_layout gives
 * them for the same T, H, E, k, I) followed by the shared expert's (every region 256-byte aligned):
 *   xq int8 [T, H] and sx fp32 [T] (per-token codes and scales of x, token order);
 *   h bf16 [T, Is] (SiLU(gate) * up); s_h fp32 [T]; hq int8 [T, Is]; o bf16 [T, H];
 *   gate fp32 [T] (sigmoid of the shared_expert_gate logit). */
typedef struct {
  w8a8_moe_ws_layout routed;
  size_t xq, sx, h, s_h, hq, o, gate;
  size_t total;
} w8a8_moe_shared_ws_layout;

/* Fills *layout for the shape (Is: the shared expert's intermediate size, a multiple of 128).
 * Returns W8A8_ERR_ARG / W8A8_ERR_UNSUPPORTED on bad shapes. */
int w8a8_moe_shared_workspace_layout(int64_t T, int64_t H, int64_t E, int k, int64_t I, int64_t Is,
                                     w8a8_moe_shared_ws_layout* layout);

/* Workspace bytes w8a8_moe_forward_shared needs for this shape (0 if the shape is rejected). */
size_t w8a8_moe_shared_workspace_size(int64_t T, int64_t H, int64_t E, int k, int64_t I, int64_t Is);

/* Defined by: "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战", section 二 2.2
 * (the shared expert is a dense path, quantised W8A8 directly, next to the packed routed experts);
 * the ignore list of the Qwen3.6-35B-A3B-w8a8 recipe (shared_expert_gate stays bf16). The pages
 * do not give how the two paths combine; the library reads it as y = routed + sigmoid(x . w_sg) *
 * shared.
 * MoE layer with a shared expert: the routed forward of w8a8_moe_forward, plus on every token
 *   g = sigmoid(x . w_sg) (bf16 inputs, fp32 sum, fp32 sigmoid), the shared expert as a dense W8A8
 *   gated MLP (per-token int8 x, int8 gate_up, dequant, SiLU(gate) * up -> bf16 h, per-row int8
 *   requantisation, int8 down, dequant -> bf16 o_s), and
 *   y[t] = bf16(fma(g[t], o_s[t], acc_t)), acc_t the fp32 accumulator of the routed combine.
 *   wsg    bf16 [H]        shared_expert_gate (nn.Linear H -> 1)
 *   wgu_s  int8 [2Is, H]   packed gate|up of the shared expert; s_gu_s fp32 [2Is]
 *   wd_s   int8 [H, Is];   s_d_s fp32 [H]
 *   workspace  at least w8a8_moe_shared_workspace_size() bytes, 256-byte aligned; it keeps the
 *              intermediates listed in w8a8_moe_shared_ws_layout after the call.
 * The other arguments and rules are those of w8a8_moe_forward; Is % 128 == 0. */
int w8a8_moe_forward_shared(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                            const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H, int64_t E,
                            int k, int64_t I, int renorm, const w8a8_bf16* wsg, const int8_t* wgu_s,
                            const float* s_gu_s, const int8_t* wd_s, const float* s_d_s, int64_t Is, void* workspace,
                            size_t workspace_bytes, w8a8_bf16* y, w8a8_stream stream);

/* w8a8_moe_forward that also records caller-created CUDA events (cudaEvent_t, may be NULL
 * entries) on `stream` at the stage boundaries, for per-kernel timing:
 *   [0] before the router, [1] before grouping + quantisation, [2] before the gate_up GEMM,
 *   [3] before the requantisation of h, [4] before the down GEMM, [5] before the combine,
 *   [6] after the combine. stage_events must point to 7 entries. */
int w8a8_moe_forward_profiled(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                              const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H,
                              int64_t E, int k, int64_t I, int renorm, void* workspace, size_t workspace_bytes,
                              w8a8_bf16* y, w8a8_stream stream, void* const* stage_events);

/* Allocation-free variant of w8a8_moe_forward (no counterpart on the pages: it only changes
 * where the scratch memory comes from).
 *
 * Some callers cannot hand this library a workspace: code on a latency-critical serving path
 * where cudaMalloc may synchronise the whole device and stall every other stream, plugins
 * whose host framework owns all device memory and lends none, and processes that run under
 * a fixed device-memory budget decided before the first request. For them this entry point
 * keeps its scratch in a buffer compiled into the library: W8A8_NOALLOC_SCRATCH_BYTES bytes
 * of device memory that every GPU loading the library holds until the process exits.
 *
 *   - Arguments and results are those of w8a8_moe_forward, without the workspace.
 *   - The call allocates and frees nothing. Shapes whose workspace (w8a8_moe_workspace_size)
 *     exceeds W8A8_NOALLOC_SCRATCH_BYTES are rejected with W8A8_ERR_UNSUPPORTED before
 *     anything is enqueued; that covers decode-sized batches (up to about 240 tokens of the
 *     Qwen3-30B-A3B shaped layer, about 120 of the Qwen3-235B-A22B shaped one), not prefill.
 *   - The first call on a device looks the buffer's address up on that device (the device
 *     must be current) and caches it with the device's context; a call in a different context
 *     of that device (after a device reset) looks it up again. Make the first call on a device
 *     before any stream capture begins. Devices with an index of 64 or more are not covered:
 *     the call returns W8A8_ERR_UNSUPPORTED there.
 *   - All calls on one device share the one buffer; each call overwrites it and resets what
 *     must start at zero. Calls whose work overlaps on the GPU (different streams without
 *     ordering between them) race on the buffer: serialise them, e.g. on one stream. The
 *     intermediates of the last call stay in the buffer but are not exposed. */
#define W8A8_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int w8a8_moe_forward_noalloc(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                             const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H,
                             int64_t E, int k, int64_t I, int renorm, w8a8_bf16* y, w8a8_stream stream);

/* Workspace bytes w8a8_linear needs (0 if the shape is rejected). */
size_t w8a8_linear_workspace_size(int64_t M, int64_t K, int64_t N, int w_format, int group);

/* Defined by: the group_0 block of the Qwen3.6-35B-A3B-w8a8 config page (int8 formats);
 * "Qwen3-235B-A22B-quantized.w8a8" shard contents (q/k/v/o projections in INT8); the
 * "Qwen3-1.7B-W4A8-V1" explainer, sections "4bit 权重" and "8bit 激活" (int4 format).
 * Dense W8A8 / W4A8 linear: y = x . W^T with per-token dynamic int8 x.
 *   W8A8_W_INT8_PER_CHANNEL: w int8 [N, K], sw fp32 [N]; y = bf16(((float)acc * s_x) * sw[n]).
 *   W8A8_W_INT4_PER_GROUP:   w uint8 [N, K/2] (packing as above), sw fp32 [N, K/group];
 *     y = bf16(acc_f * s_x) with acc_f = sum over groups g in order of (float)acc_g * sw[n, g],
 *     acc_g the int32 sum of group g (fp32 products and sums).
 *   x bf16 [M, K]; workspace of w8a8_linear_workspace_size() bytes; y bf16 [M, N].
 * K % 128 == 0, N % 128 == 0, group == 128 for the int4 format. */
int w8a8_linear(const w8a8_bf16* x, const void* w, const float* sw, int w_format, int group, int64_t M,
                int64_t K, int64_t N, void* workspace, size_t workspace_bytes, w8a8_bf16* y, w8a8_stream stream);

/* The GEMM of w8a8_linear on activations already quantised per token (for example by
 * w8a8_quant_act_per_token, or by a producer that emits int8 codes directly):
 *   xq int8 [M, K], sx fp32 [M] (per-token scales); w, sw, w_format, group, y as w8a8_linear.
 * Same shape rules and results as w8a8_linear given the same xq and sx; needs no workspace. */
int w8a8_linear_prequant(const int8_t* xq, const float* sx, const void* w, const float* sw, int w_format, int group,
                         int64_t M, int64_t K, int64_t N, w8a8_bf16* y, w8a8_stream stream);

/* Defined by: section 六 of "Qwen3-Next-80B-A3B-Instruct 在 AMCT 中的 MoE 混合注意力量化适配实战",
 * the "MXFP A8w8" row of its accuracy table (the format is named there and nothing more; it is
 * read as the OCP Microscaling FP8 format).
 * MXFP8 quantisation of bf16 rows along K, in blocks of 32 consecutive values:
 *   E = floor(log2(max |v| of the block)) - 8, clamped to [-127, 127] (-127 for a block of zeros);
 *   scales[r, b] = E + 127 (an E8M0 byte: the block's scale is 2^E);
 *   codes[r, k] = the FP8 E4M3 byte of v * 2^-E: nearest, ties to even, magnitudes above 448
 *   saturating to 448, the sign kept when the value rounds to zero.
 * Used for the weights of a layer (once, per output channel) and, inside w8a8_mxfp8_linear, for
 * its activations (per token, at every call).
 *   x bf16 [R, K] (16-byte aligned), codes uint8 [R, K] (8-byte aligned), scales uint8 [R, K/32];
 *   all device memory owned by the caller. K % 32 == 0 (else W8A8_ERR_UNSUPPORTED). */
int w8a8_mxfp8_quantize(const w8a8_bf16* x, int64_t R, int64_t K, uint8_t* codes, uint8_t* scales,
                        w8a8_stream stream);

/* Workspace bytes w8a8_mxfp8_linear needs (0 if the shape is rejected). */
size_t w8a8_mxfp8_linear_workspace_size(int64_t M, int64_t K, int64_t N);

/* Defined by: the same row of the same table (MXFP8 A8W8: both operands in MXFP8).
 * Dense MXFP8 A8W8 linear: x is quantised to MXFP8 per token (w8a8_mxfp8_quantize), then the
 * block-scaled FP8 MMA of the tensor cores (tcgen05 kind::mxf8f6f4, one E8M0 scale per 32 values of
 * K on both operands) sums the products of the dequantised values in fp32:
 *   y[m, n] = bf16(sum_k (P_x[m,k] 2^Ex[m,k/32]) (P_w[n,k] 2^Ew[n,k/32])),
 * in the tensor core's own summation order (within (K - 1) * 2^-24 * sum_k |products| of the exact
 * sum before the bf16 rounding).
 *   x bf16 [M, K] (16-byte aligned); w_codes uint8 [N, K] (16-byte aligned) and w_scales uint8
 *   [N, K/32] (4-byte aligned) from w8a8_mxfp8_quantize; workspace of
 *   w8a8_mxfp8_linear_workspace_size() bytes (256-byte aligned; it receives x's codes at offset 0
 *   and its scales after them, 256-byte aligned); y bf16 [M, N].
 * K % 128 == 0, N % 128 == 0 (else W8A8_ERR_UNSUPPORTED). */
int w8a8_mxfp8_linear(const w8a8_bf16* x, const uint8_t* w_codes, const uint8_t* w_scales, int64_t M, int64_t K,
                      int64_t N, void* workspace, size_t workspace_bytes, w8a8_bf16* y, w8a8_stream stream);

/* The GEMM of w8a8_mxfp8_linear on activations already in MXFP8 (for example from
 * w8a8_mxfp8_quantize): x_codes uint8 [M, K] (16-byte aligned), x_scales uint8 [M, K/32] (4-byte
 * aligned); the weights, y and the shape rules as w8a8_mxfp8_linear. Needs no workspace. */
int w8a8_mxfp8_linear_prequant(const uint8_t* x_codes, const uint8_t* x_scales, const uint8_t* w_codes,
                               const uint8_t* w_scales, int64_t M, int64_t K, int64_t N, w8a8_bf16* y,
                               w8a8_stream stream);

/* Defined by: the "MXFP A8w4" row of the same table (MXFP8 activations, MXFP4 weights), read as
 * the OCP Microscaling FP4 format for the weights.
 * MXFP4 quantisation of bf16 rows along K, for the weights of an MXFP A8W4 layer (once, per output
 * channel): per block of 32 values E = floor(log2 max|v|) - 2 (clamped to [-127, 127], -127 for a
 * zero block), scale byte E + 127 (E8M0), elements E2M1(v * 2^-E) rounded to nearest with ties to
 * even and saturated at 6, the sign kept at zero; two codes per byte, element 2i in the low nibble.
 *   w bf16 [R, K] (16-byte aligned), packed uint8 [R, K/2] (4-byte aligned), scales uint8 [R, K/32];
 *   all device memory owned by the caller. K % 32 == 0 (else W8A8_ERR_UNSUPPORTED). */
int w8a8_mxfp4_quantize(const w8a8_bf16* w, int64_t R, int64_t K, uint8_t* packed, uint8_t* scales,
                        w8a8_stream stream);

/* Defined by: the same row (MXFP A8W4).
 * Dense MXFP A8W4 linear: x is quantised to MXFP8 per token (as in w8a8_mxfp8_linear), then the
 * block-scaled MMA multiplies its E4M3 codes by the E2M1 weight codes, one E8M0 scale per 32
 * values of K on both operands, summing in fp32:
 *   y[m, n] = bf16(sum_k (P_x[m,k] 2^Ex[m,k/32]) (P_w[n,k] 2^Ew[n,k/32])),
 * within the same summation bound as w8a8_mxfp8_linear.
 *   x bf16 [M, K] (16-byte aligned); w_packed uint8 [N, K/2] (32-byte aligned) and w_scales uint8
 *   [N, K/32] (4-byte aligned) from w8a8_mxfp4_quantize; workspace of
 *   w8a8_mxfp8_linear_workspace_size() bytes (256-byte aligned; x's MXFP8 codes at offset 0 and
 *   its scales after them, 256-byte aligned); y bf16 [M, N].
 * K % 128 == 0, N % 128 == 0 (else W8A8_ERR_UNSUPPORTED). */
int w8a8_mxfp_a8w4_linear(const w8a8_bf16* x, const uint8_t* w_packed, const uint8_t* w_scales, int64_t M,
                          int64_t K, int64_t N, void* workspace, size_t workspace_bytes, w8a8_bf16* y,
                          w8a8_stream stream);

/* The GEMM of w8a8_mxfp_a8w4_linear on activations already in MXFP8: x_codes uint8 [M, K]
 * (16-byte aligned), x_scales uint8 [M, K/32] (4-byte aligned); the weights, y and the shape rules
 * as w8a8_mxfp_a8w4_linear. Needs no workspace. */
int w8a8_mxfp_a8w4_linear_prequant(const uint8_t* x_codes, const uint8_t* x_scales, const uint8_t* w_packed,
                                   const uint8_t* w_scales, int64_t M, int64_t K, int64_t N, w8a8_bf16* y,
                                   w8a8_stream stream);

/* Exact integer GEMM on the tensor cores: c[m, n] = sum_k a[m, k] * b[n, k] in int32: the
 * int8 x int8 product every W8A8 Linear of the group_0 scheme accumulates before its scales.
 *   a int8 [M, K], b int8 [N, K], c int32 [M, N];  K % 128 == 0, N % 128 == 0. */
int w8a8_gemm_s8s8s32(const int8_t* a, const int8_t* b, int32_t* c, int64_t M, int64_t N, int64_t K,
                      w8a8_stream stream);

/* Test hook for the certified SiLU evaluation: writes to *max_ulp (device memory, one uint32)
 * the largest distance, in units in the last place, between the hardware's approximate
 * reciprocal (rcp.approx.ftz.f32) and the correctly rounded reciprocal over the `count` fp32 bit
 * patterns starting at `first_bits`. They must be positive normal numbers with normal
 * reciprocals ([2^-126, 2^126)), else W8A8_ERR_ARG. The gated-activation epilogue of the
 * CTA-pair gate_up GEMM relies on this distance being at most 2. */
int w8a8_debug_rcp_approx_ulp(uint32_t first_bits, uint32_t count, unsigned int* max_ulp, w8a8_stream stream);

/* Test hook for the certified SiLU evaluation: writes to *max_ulp (device memory, one uint32)
 * the largest distance, in units in the last place, between the hardware's approximate base-2
 * exponential (ex2.approx.ftz.f32) and 2^x computed in double precision and rounded to fp32, over
 * the `count` fp32 bit patterns starting at `first_bits`. They must share one sign and satisfy
 * |x| < 126 (2^x normal), else W8A8_ERR_ARG. The gated-activation epilogue of the CTA-pair
 * gate_up GEMM relies on this distance being at most 3. */
int w8a8_debug_ex2_approx_ulp(uint32_t first_bits, uint32_t count, unsigned int* max_ulp, w8a8_stream stream);

/* Test hook for the bounded waits: launches one CTA that waits on an mbarrier phase nothing
 * completes; after `timeout_ns` the wait gives up and sets the device error word, which the
 * next w8a8_check_status() reports as W8A8_ERR_DEVICE. The context stays usable.
 * Every wait inside the library's kernels is bounded the same way: a single wait (an mbarrier
 * phase, a grid barrier) that has not completed 2 s after it began (or the number of
 * milliseconds in the environment variable W8A8_WAIT_TIMEOUT_MS, read once per process) gives
 * up. The bound applies to each wait on its own, not to the lifetime of a kernel. */
int w8a8_debug_wait_timeout(uint64_t timeout_ns, w8a8_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H_ */
