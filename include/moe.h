/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of one sparse
 * Mixture-of-Experts layer:
 *
 *   router logits -> softmax over all experts -> top-k -> dispatch (permute)
 *   -> per-expert SwiGLU feed-forward -> gate-weighted combine (unpermute).
 *
 * Passages (page title, then section):
 *   [P2] "Kimi K3: The Open Model That Just Cornered the AI Frontier",
 *        section "Mixture-of-Experts with Dynamic Load Balancing", gating code:
 *        logits from one gate projection, softmax over the expert axis, top-k
 *        of the probabilities, values and indices returned as they are.
 *   [P3] "Kimi K3: Open Frontier Intelligence", section "Operational Execution
 *        Flow": tokens are dispatched to their active routed experts and the
 *        routed output is the probability-weighted sum of the selected experts'
 *        outputs; the experts use a GLU feed-forward whose SwiGLU regime the
 *        page names.
 *   Model-card shapes: 384 experts top-8 ("Kimi K3: What Open-Source Frontier
 *   Models Reveal About RL Scaling for Reasoning", section "The Architecture:
 *   MoE, Latent Attention, and Massive Context"), 256 top-4 ([P2]), 896
 *   top-16 and d_model 7168 ([P3]).
 *
 * Conventions for every entry point
 *   - Every pointer is a DEVICE pointer owned by the caller, unless stated.
 *     The library never allocates, frees or synchronises; every call only
 *     enqueues kernels on `stream` and returns.
 *   - All tensors are dense, row-major, with no padding between rows.
 *     bf16 tensors are passed as `const moe_bf16_t*` (the 16-bit patterns).
 *     x, W_gate_up, W_down, x_perm, h, y_perm and out must be 16-byte aligned.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns a status other than MOE_OK and launches nothing.
 *   - MOE_ERR_CUDA means a launch failed (cudaGetLastError after the launches).
 *   - Kernels that wait on hardware barriers wait for a bounded time; if a
 *     wait runs out they record a code in a per-device error word and return
 *     early (outputs are then undefined). moe_get_device_error() reads it.
 *   - Sizes: T >= 1 tokens, d model width, E experts, 1 <= k <= min(E, 16)
 *     selected experts per token, f expert hidden width. d and f must be
 *     multiples of 64; E <= 1024; T * k < 2^31; d, f <= 32768.
 */
#ifndef MOE_B200_MOE_H_
#define MOE_B200_MOE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h> /* cudaStream_t */

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t; /* bfloat16 bit pattern */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, size out of range, misalignment */
  MOE_ERR_UNSUPPORTED = 2, /* valid but beyond the library's limits (k > 16, E > 1024, ...) */
  MOE_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than required */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE = 5       /* a kernel recorded an error (see moe_get_device_error) */
} moe_status_t;

/* Human-readable name of a status. Never NULL. */
const char* moe_status_string(moe_status_t status);

/* Maximum k and E supported by the register top-k. */
#define MOE_MAX_TOPK 16
#define MOE_MAX_EXPERTS 1024

/* ---------------------------------------------------------------- router --
 * moe_route: steps 1-3 of the pass ([P2] gating code).
 *   logits[t, e] = sum_i x[t, i] * W_router[i, e]  (+ router_bias[e])
 *     computed in fp32 (x widened exactly from bf16) in a fixed order: fma
 *     inside consecutive chunks of 128 input indices, chunk partials added in
 *     ascending chunk order, bias added last. The order makes the routing
 *     reproducible bit for bit.
 *   probs[t, :] = softmax(logits[t, :]) over all E experts (fp32).
 *   topk_idx[t, 0..k-1]: the experts with the k largest logits, descending;
 *     equal logits go to the lower expert index.
 *   topk_w[t, j] = probs[t, topk_idx[t, j]], NOT renormalised.
 * Inputs:  x [T, d] bf16; W_router [d, E] fp32; router_bias [E] fp32 or NULL.
 * Outputs: topk_idx [T, k] int32; topk_w [T, k] fp32.
 * Scratch: workspace of at least moe_route_workspace_size(T, d, E) bytes,
 *   256-byte aligned (holds fp32 logits or per-chunk partial sums; for T <= 16
 *   and E % 4 == 0 also the final logits and the completion counters of the
 *   single-launch few-token router, which the call clears itself; for
 *   T >= 256 the tensor-core screen's operands and partial sums).
 */
size_t moe_route_workspace_size(int T, int d, int E);
moe_status_t moe_route(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                       int T, int d, int E, int k,
                       int32_t* topk_idx, float* topk_w,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* --------------------------------------------------------------- permute --
 * moe_permute: step 4, dispatch ([P3] tokens are dispatched to their routed
 * experts). A stable counting sort of the T*k (token, slot) pairs by expert:
 *   expert_offsets[e] = number of pairs routed to experts < e  ([E+1] int32,
 *     expert_offsets[E] = T*k);
 *   rows expert_offsets[e] .. expert_offsets[e+1]-1 hold the tokens routed to
 *     expert e in ascending token order: perm_token[row] = token ([T*k] int32);
 *   inv_perm[t*k + j] = row of the pair (t, j)  ([T, k] int32);
 *   x_perm[row, :] = x[perm_token[row], :]  ([T*k, d] bf16; may be NULL to
 *     skip the row copy).
 * Inputs: x [T, d] bf16 (may be NULL when x_perm is NULL); topk_idx [T, k].
 * Scratch: moe_permute_workspace_size(T, E, k) bytes, 256-byte aligned.
 */
size_t moe_permute_workspace_size(int T, int E, int k);
moe_status_t moe_permute(const moe_bf16_t* x, const int32_t* topk_idx,
                         int T, int d, int E, int k,
                         int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm,
                         moe_bf16_t* x_perm,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ expert FFN --
 * moe_expert_ffn: step 5, every expert's SwiGLU feed-forward on its rows.
 * For expert e and each row r in expert_offsets[e] .. expert_offsets[e+1]-1:
 *   g = x_perm[r, :] @ W_gate_up[e][:, 0:f]      (gate half)
 *   u = x_perm[r, :] @ W_gate_up[e][:, f:2f]     (up half)
 *   h[r, :] = SiLU(g) * u, SiLU(a) = a / (1 + exp(-a))   -> bf16 [Tk, f]
 *   y_perm[r, :] = h[r, :] @ W_down[e]                    -> bf16 [Tk, d]
 * bf16 operands on the tcgen05 tensor cores, fp32 accumulation, fp32
 * epilogue, round-to-nearest-even to bf16.
 * Inputs: x_perm [Tk, d] bf16; expert_offsets [E+1] int32 (device; read on the
 *   device, no host sync); W_gate_up [E, d, 2f] bf16; W_down [E, f, d] bf16.
 * Outputs: h [Tk, f] bf16 (also the operand of the second GEMM); y_perm [Tk, d].
 * Scratch: moe_expert_ffn_workspace_size(Tk, E) bytes, 256-byte aligned: the
 *   GEMM tile schedules and, when min(E, Tk) <= 592 (few output tiles, where
 *   the GEMMs split (tile, K-block) work evenly over the SMs), fp32 partial
 *   tiles and completion counters. The split follows from the shapes and the
 *   partial sums are added in ascending K order, so results are deterministic.
 */
size_t moe_expert_ffn_workspace_size(int Tk, int E);
moe_status_t moe_expert_ffn(const moe_bf16_t* x_perm, const int32_t* expert_offsets,
                            const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down,
                            int Tk, int d, int E, int f,
                            moe_bf16_t* h, moe_bf16_t* y_perm,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------- unpermute --
 * moe_unpermute: step 6, the gate-weighted combine ([P3] the routed output is
 * the probability-weighted sum of the selected experts' outputs):
 *   out[t, :] = sum_{j=0..k-1} topk_w[t, j] * y_perm[inv_perm[t*k + j], :]
 * accumulated in fp32 in ascending j, stored bf16 [T, d].
 * Needs no scratch.
 */
moe_status_t moe_unpermute(const moe_bf16_t* y_perm, const int32_t* inv_perm, const float* topk_w,
                           int T, int d, int k, moe_bf16_t* out, cudaStream_t stream);

/* --------------------------------------------------------------- forward --
 * moe_forward: the whole pass (route, permute, expert FFN, unpermute) on one
 * stream, with no host synchronisation. All intermediates are carved from
 * `workspace` (at least moe_forward_workspace_size(T, d, E, k, f) bytes,
 * 256-byte aligned). out [T, d] bf16.
 * Launch shapes: T <= 32 runs both expert GEMMs as one cooperative launch
 * (its own K split, so its sums may differ from moe_expert_ffn's in rounding
 * order); T = 1 with d <= 8192 runs the whole layer as one cooperative launch
 * (after an 8-byte memset of its barrier counts), bit-identical to the
 * separate stages that moe_forward_timed runs.
 */
size_t moe_forward_workspace_size(int T, int d, int E, int k, int f);
moe_status_t moe_forward(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                         const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down,
                         int T, int d, int E, int k, int f,
                         moe_bf16_t* out,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* moe_forward_timed: moe_forward that also records CUDA events around its
 * kernel groups on `stream`, for live per-kernel timing. `events` holds
 * 2 * MOE_TIMED_STAGES caller-created events (cudaEventCreate); stage i is
 * bracketed by events[2*i] and events[2*i+1]:
 *   0 router (logits + softmax/top-k)   1 dispatch (histogram, scan, scatter,
 *   row copy, GEMM tile schedule)       2 gate/up grouped GEMM (one kernel)
 *   3 down grouped GEMM (one kernel)    4 combine (one kernel)
 * Same arguments, results and errors as moe_forward otherwise; events == NULL
 * is MOE_ERR_INVALID_ARG. The stages always run as separate launches (for
 * T = 1 the router, the feed-forward and the combine, where moe_forward runs
 * one launch).
 */
#define MOE_TIMED_STAGES 5
moe_status_t moe_forward_timed(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                               const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down,
                               int T, int d, int E, int k, int f,
                               moe_bf16_t* out,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream,
                               cudaEvent_t* events);

/* moe_forward_host: moe_forward with x and out in HOST memory -- the call a
 * host program makes when its activations live on the CPU side. On `stream`,
 * in this order: one cudaMemcpyAsync of x_host [T, d] bf16 into a staging
 * buffer at the start of `workspace`, the whole pass (exactly the kernels of
 * moe_forward), and one cudaMemcpyAsync of the result into out_host [T, d].
 * Returns once that work is enqueued; out_host holds the result when `stream`
 * has run it (synchronise the stream, or an event recorded after the call).
 * x_host must stay unchanged until then.
 * x_host and out_host should be page-locked (cudaHostAlloc/cudaHostRegister):
 * then the copies run asynchronously, and calls on two streams with two
 * workspaces overlap one call's copies with the other's kernels. Pageable
 * buffers work too, but the copies then run synchronously with the host.
 * Weights (and the bias) are device pointers, as in moe_forward.
 * Workspace: moe_forward_host_workspace_size(T, d, E, k, f) bytes, 256-byte
 * aligned = two [T, d] bf16 staging buffers (each rounded up to 256 bytes)
 * followed by moe_forward's workspace.
 * Errors: as moe_forward; a device (or managed) pointer for x_host or
 * out_host is MOE_ERR_INVALID_ARG, a failed copy is MOE_ERR_CUDA.
 */
size_t moe_forward_host_workspace_size(int T, int d, int E, int k, int f);
moe_status_t moe_forward_host(const moe_bf16_t* x_host, const float* W_router, const float* router_bias,
                              const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down,
                              int T, int d, int E, int k, int f,
                              moe_bf16_t* out_host,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------- allocation-free router --
 * moe_route_noalloc: moe_route for callers that cannot allocate device memory
 * -- for example code running inside a host framework that owns every device
 * allocation, or a serving loop that must not call into an allocator between
 * steps. The pages have no counterpart to this entry point; it exists only for
 * such callers. The caller still passes the inputs and outputs; the scratch
 * that moe_route takes as `workspace` is instead a fixed array inside the
 * library, MOE_ROUTE_NOALLOC_SCRATCH_BYTES (4 MiB) per device, held by every
 * GPU that loads the library until the process exits.
 * Same arguments (minus the workspace), results and errors as moe_route, plus:
 *   - sizes whose scratch, moe_route_workspace_size(T, d, E), exceeds
 *     MOE_ROUTE_NOALLOC_SCRATCH_BYTES return MOE_ERR_UNSUPPORTED and launch
 *     nothing (for d = 7168, E = 896 that is T > 20);
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on that device;
 *   - every call on a device shares the one array: calls that overlap on the
 *     GPU (different streams, no ordering between them) race and give
 *     undefined results. Nothing needs clearing between calls, because each
 *     call writes every scratch element it reads before reading it.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (4u << 20)
moe_status_t moe_route_noalloc(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                               int T, int d, int E, int k,
                               int32_t* topk_idx, float* topk_w, cudaStream_t stream);

/* ------------------------------------------------------- MX quantisation --
 * The serving format of [P3] section "Systems Optimization, Load Balancing,
 * and Post-Training Alignment": MXFP4 expert weights with MXFP8 activations.
 * The page names the formats only; the reading taken is the published OCP
 * Microscaling (MX) format. Blocks of 32 consecutive values along the
 * reduction axis share a scale 2^s, stored as the E8M0 byte s + 127, with
 * s = floor(log2(max |v| of the block)) - emax clamped to [-127, 127]
 * (emax = 2 for E2M1, 8 for E4M3; an all-zero block takes s = -127). Each
 * element is v / 2^s rounded to the nearest element value (ties to the even
 * code), saturating at the largest finite magnitude (6 for E2M1, 448 for
 * E4M3), with the sign bit of v (also when the magnitude rounds to 0).
 * Codes are one per byte: E2M1 in bits 3..0 (bit 3 the sign), E4M3 in the
 * whole byte (bit 7 the sign; NaN codes are never produced).
 * Inputs must be finite (a NaN or infinity gives an unspecified code).
 * Neither call needs scratch; both only enqueue one kernel on `stream`.
 *
 * moe_mxfp8_quantize: x [rows, cols] bf16 (cols % 32 == 0, x 16-byte
 * aligned), blocks along each row: codes [rows, cols] (16-byte aligned),
 * scales [rows, cols / 32]. rows >= 1, 32 <= cols <= 2^20.
 */
moe_status_t moe_mxfp8_quantize(const moe_bf16_t* x, int rows, int cols,
                                uint8_t* codes, uint8_t* scales, cudaStream_t stream);

/* moe_mxfp4_quantize: w [K, N] bf16 (N contiguous; an expert's W_gate_up is
 * [d, 2f], its W_down [f, d]), K % 32 == 0, blocks along K for each column:
 * codes [K, N], scales [K / 32, N]. 32 <= K <= 2^20, 1 <= N <= 2^20.
 * A whole stack of experts [E, K, N] is one call with K' = E * K (every
 * block then lies inside one expert, since K % 32 == 0).
 */
moe_status_t moe_mxfp4_quantize(const moe_bf16_t* w, int K, int N,
                                uint8_t* codes, uint8_t* scales, cudaStream_t stream);

/* ------------------------------------------------ MX expert feed-forward --
 * The layer with its experts in the serving format above: MXFP4 expert
 * weights, MXFP8 token activations (x and the SwiGLU output h), on the
 * block-scaled tensor cores. Routing, dispatch and combine are those of
 * moe_forward (bit-identical routing); only the expert GEMMs change.
 * Requires d % 256 == 0 and f % 128 == 0 (128 <= f <= 32768).
 *
 * moe_mx_expert_bytes: sizes of the four packed arrays for E experts of
 * width d and hidden width f (n = E * d * f):
 *   wq_gate_up n bytes, sf_gate_up n / 16, wq_down n / 2, sf_down n / 32.
 * moe_mx_pack_experts: quantises W_gate_up [E, d, 2f] and W_down [E, f, d]
 * (bf16, as moe_forward takes them) with the MXFP4 rule above, blocks of 32
 * along each matrix's reduction axis (d, resp. f), into
 *   wq_*: the E2M1 codes of each output feature's column, the reduction axis
 *         contiguous, two codes per byte (even index in the low nibble):
 *         [E][2f][d / 2] and [E][d][f / 2];
 *   sf_*: the E8M0 scales grouped in 512-byte atoms, one per 128 output
 *         features x 128 reduction elements: [E][2f / 128][d / 128][512]
 *         and [E][d / 128][f / 128][512]; feature m and block b of an atom
 *         at byte 16 * (m % 32) + 4 * (m / 32) + b.
 *   wq_* 32-byte aligned, sf_* 16-byte aligned. One-time preparation of the
 *   weights; enqueues two kernels on `stream`.
 * moe_forward_mx: as moe_forward, with the packed experts in place of
 *   W_gate_up / W_down. x takes an MXFP8 round trip along d before the
 *   gate/up GEMM and h one along f before the down GEMM (the arithmetic of the
 *   MX oracle); y is accumulated in fp32 and stored bf16. Workspace:
 *   moe_forward_mx_workspace_size(T, d, E, k, f) bytes, 256-byte aligned.
 */
moe_status_t moe_mx_expert_bytes(int E, int d, int f, size_t* wq_gate_up, size_t* sf_gate_up,
                                 size_t* wq_down, size_t* sf_down);
moe_status_t moe_mx_pack_experts(const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, int E, int d, int f,
                                 uint8_t* wq_gate_up, uint8_t* sf_gate_up, uint8_t* wq_down, uint8_t* sf_down,
                                 cudaStream_t stream);
size_t moe_forward_mx_workspace_size(int T, int d, int E, int k, int f);
moe_status_t moe_forward_mx(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                            const uint8_t* wq_gate_up, const uint8_t* sf_gate_up,
                            const uint8_t* wq_down, const uint8_t* sf_down,
                            int T, int d, int E, int k, int f,
                            moe_bf16_t* out,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------- Quantile Balancing --
 * The per-expert bias update of [P3] section "Systems Optimization, Load
 * Balancing, and Post-Training Alignment" (QB): biases from the (1 - k/n)-
 * quantile over tokens of the margins s[t,e] - alpha_t, alpha_t the cutoff of
 * top-(k+1) routing, recovered from per-expert binned histograms that
 * data-parallel ranks add up with one integer all-reduce. The page's update
 * formula is garbled; the reading taken, the dual step of the
 * balanced-assignment LP the page names, is:
 *   alpha_t = (k+1)-th largest of s[t,e] + b[e];
 *   beta_e  = the ceil(m k / n)-th largest margin s[t,e] - alpha_t of expert e
 *             (m tokens over all ranks, n = E experts);
 *   b_new[e] = -beta_e, beta_e taken at the lower edge of its histogram bin.
 * All arithmetic is fp32 with every operation rounded as written:
 *   v = s + b, mu = s - alpha, t = mu - lo, bin = !(t >= 0) ? 0 : (t * inv_w
 *   >= B ? B - 1 : trunc(t * inv_w)), inv_w = fp32(B) / fp32(hi - lo); a NaN
 *   margin (from a NaN logit, or infinite ones that cancel) counts in bin 0.
 *
 * moe_router_logits: the router logits s = x W_router (+ bias) [T, E] fp32 in
 *   the canonical order of moe_route (bit-identical to the logits it selects
 *   on), for every expert. No scratch. T <= 4194240 (64 x 65535).
 * moe_qb_histogram: from logits [T, E] and the current biases (NULL: zero),
 *   writes alpha [T] and ADDS this batch's margin counts into H [E][bins]
 *   (uint64; zero it before the first batch, then all-reduce it over ranks).
 *   2 <= E <= 1024, 1 <= k < E, k <= 16, 1 <= bins <= 1536, lo < hi finite.
 * moe_qb_bias: from the (summed) H and m_total, the number of tokens each row
 *   of H counts, writes bin_out [E] (the quantile's bin: the highest bin whose
 *   count from the top reaches ceil(m_total k / E), or 0) and bias_out [E] =
 *   -(lo + bin * w), w = fp32(hi - lo) / fp32(bins), in fp32.
 * All three only enqueue kernels on `stream`.
 */
moe_status_t moe_router_logits(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                               int T, int d, int E, float* logits, cudaStream_t stream);
moe_status_t moe_qb_histogram(const float* logits, const float* bias, int T, int E, int k,
                              float lo, float hi, int bins, float* alpha, uint64_t* H, cudaStream_t stream);
moe_status_t moe_qb_bias(const uint64_t* H, int E, int bins, float lo, float hi, int64_t m_total, int k,
                         int32_t* bin_out, float* bias_out, cudaStream_t stream);

/* ----------------------------------------------- expert parallelism --
 * [P3] section "Systems Optimization, Load Balancing, and Post-Training
 * Alignment" (its expert-parallel scheme): the routed experts are split over
 * ranks, and each rank's dispatched token rows go to the rank that owns their
 * expert and come back after the expert feed-forward. The exchanges are the
 * caller's all-to-all collectives (NCCL); on either side of them the rows have
 * to be put in the order the next step reads, which is a row gather.
 *
 * moe_gather_rows: out[i, :] = src[rows[i], :] for 0 <= i < n_out (bf16 rows
 *   of width d; src [n_src, d], out [n_out, d], row-major, 16-byte aligned,
 *   d % 8 == 0). rows[i] = -1 writes a zero row (the padding of a
 *   fixed-capacity exchange buffer); any other index outside [0, n_src)
 *   writes a zero row and records MOE_DEVERR_BAD_ROUTE in the error word.
 *   Needs no scratch; n_out = 0 enqueues nothing.
 */
moe_status_t moe_gather_rows(const moe_bf16_t* src, int64_t n_src, const int32_t* rows, int64_t n_out, int d,
                             moe_bf16_t* out, cudaStream_t stream);

/* --------------------------------------------------- Stable LatentMoE --
 * [P3] section "Operational Execution Flow": two full-width shared experts
 * act on x; the routed path projects x down to a latent z = x W_dn of width l
 * (3584 on the page), the k routed experts chosen by the router (on x, as in
 * moe_route) act on z, their probability-weighted sum u passes an explicit
 * RMSNorm, and W_up brings it back to width d. The experts' GLU is SiTU-GLU,
 * a soft-capped SwiGLU with beta1 = 4, beta2 = 25 on the page and
 * |SiTU-GLU| <= beta1 beta2. The page lost the formulas; readings taken:
 *   SiTU-GLU(g, v) = beta1 tanh(SiLU(g) / beta1) * beta2 tanh(v / beta2);
 *   out = sum_s S_s(x) + RMSNorm(u) W_up, RMSNorm(u) = gamma u / sqrt(mean(u^2) + eps).
 *
 * moe_latent_forward: x [T, d] bf16; W_router [d, E] fp32, router_bias [E] or
 *   NULL; W_dn [d, l], W_up [l, d] bf16; routed W_gate_up [E, l, 2f] (columns
 *   0..f-1 gate, f..2f-1 the second factor), W_down [E, f, l] bf16; gamma [l]
 *   fp32 or NULL (ones); shared Ws_gate_up [S, d, 2fs], Ws_down [S, fs, d]
 *   bf16 (S = 0: none, both may be NULL); act 0 SwiGLU, 1 SiTU-GLU with
 *   beta1, beta2 > 0; eps >= 0. out [T, d] bf16. Intermediates (z, the
 *   routed rows, h, y, RMSNorm(u), the shared experts' outputs) are carved
 *   from `workspace` (moe_latent_workspace_size bytes, 256-byte aligned) and
 *   rounded to bf16 between the GEMMs; the routed sum, the RMSNorm and the
 *   final sum are fp32. d, l, f, fs multiples of 64; l <= 8192; S <= 8;
 *   other limits as moe_forward. Asynchronous on `stream`, no host sync.
 */
size_t moe_latent_workspace_size(int T, int d, int l, int E, int k, int f, int S, int fs);
moe_status_t moe_latent_forward(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                                const moe_bf16_t* W_dn, const moe_bf16_t* W_up,
                                const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, const float* gamma,
                                const moe_bf16_t* Ws_gate_up, const moe_bf16_t* Ws_down,
                                int T, int d, int l, int E, int k, int f, int S, int fs,
                                int act, float beta1, float beta2, float eps,
                                moe_bf16_t* out, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ diagnostics --
 * moe_get_device_error: reads (and, if clear != 0, resets) the error word of
 * the CURRENT device. *code is 0 when no kernel recorded an error, otherwise
 * one of MOE_DEVERR_*. This call synchronises the device (it is a debug aid,
 * not part of the hot path). Returns MOE_ERR_CUDA if the read fails,
 * MOE_ERR_DEVICE if *code != 0, MOE_OK otherwise.
 */
#define MOE_DEVERR_NONE 0u
#define MOE_DEVERR_WAIT_TIMEOUT_PRODUCER 1u /* TMA producer gave up waiting for a free stage */
#define MOE_DEVERR_WAIT_TIMEOUT_MMA 2u      /* MMA issuer gave up waiting for operands/accumulator */
#define MOE_DEVERR_WAIT_TIMEOUT_EPILOGUE 3u /* epilogue gave up waiting for an accumulator */
#define MOE_DEVERR_SELFTEST_TIMEOUT 4u      /* moe_selftest_wait_timeout fired as intended */
#define MOE_DEVERR_BAD_ROUTE 5u             /* an expert index outside [0, E) reached the dispatch */
#define MOE_DEVERR_WAIT_TIMEOUT_ROUTER 6u   /* few-token router gave up waiting for its W tile */
#define MOE_DEVERR_WAIT_TIMEOUT_DEPENDENCY 7u /* one-launch feed-forward gave up waiting for an expert's h rows */
#define MOE_DEVERR_INDEX_CHECK 8u           /* index-checking build only: a row or expert offset out of range, skipped */
moe_status_t moe_get_device_error(uint32_t* code, int clear);

/* moe_selftest_wait_timeout: launches one tiny kernel that waits, with a
 * limit of `timeout_us` microseconds (1..1000000), on a shared-memory barrier
 * that nothing ever signals, then records MOE_DEVERR_SELFTEST_TIMEOUT and
 * returns. It checks that bounded waits end and report an error instead of
 * hanging; it faults nothing. Asynchronous on `stream`.
 */
moe_status_t moe_selftest_wait_timeout(int timeout_us, cudaStream_t stream);

/* Library version (major * 10000 + minor * 100 + patch). */
int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H_ */
