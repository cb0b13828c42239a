/*
 * moe.h - C ABI of libmoe.so: one block-quantized, top-k routed Mixture-of-
 * Experts FFN layer on an NVIDIA B200 (sm_100a).
 *
 * The layer (sources: the "Strata Coder deep-dive" page, sections 1-3, and the
 * "Coder benchmark record" page, "why Coder is fast" and "expert profile file"
 * sections):
 *   - each token of hidden size H is routed to top_k of the E experts of a
 *     layer (48 layers x 512 experts, or 256 after pruning; top_k = 10);
 *   - an expert is three block-quantized projections, gate and up [I, H] and
 *     down [H, I], each with its own bit width (2 or 4), held in an expert
 *     arena addressed per (layer, expert);
 *   - routing counts per (layer, expert) accumulate into a histogram whose
 *     ranking is the expert profile.
 * Computation, per token t:
 *   l_e   = x_t . W_r[e] + b_e                      (router logits)
 *   S_t   = the top_k experts by (l desc, e asc)    (bit-exact vs fp64 math)
 *   w_j   = softmax over the chosen logits
 *   y_e   = W_d (silu(W_g x_t) * (W_u x_t))         (SwiGLU expert)
 *   out_t = (residual ? x_t : 0) + sum_j w_j y_{S_t[j]}   rounded to bf16.
 * Dequantised weight: scale_fp16[row][c/32] * (code - 2^(bits-1)).
 *
 * Conventions for every entry point:
 *   - Pointers marked (device) are caller-owned device memory, (host) are
 *     host memory.  The library allocates nothing on any call path.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Device work
 *     is enqueued asynchronously on it; the call returns once it is enqueued.
 *   - Return value: MOE_OK or a negative MOE_ERR_* code.  Errors found on the
 *     host (arguments, shapes, workspace) launch nothing.  Errors found on the
 *     device (a selected expert without a valid slot, a bounded wait that
 *     expired) are latched in a per-device status word read by
 *     moe_last_device_error().
 *   - x and out must not overlap.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_ARG (-1)      /* null or misaligned pointer, overlapping x/out  */
#define MOE_ERR_SHAPE (-2)    /* H, I, block or bit widths not supported        */
#define MOE_ERR_RANGE (-3)    /* T, E, top_k or layer outside its bound         */
#define MOE_ERR_WS (-4)       /* workspace smaller than moe_workspace_bytes()   */
#define MOE_ERR_CUDA (-5)     /* a CUDA launch or query failed                  */
#define MOE_ERR_SLOT (-6)     /* a selected expert had slot -1 or >= n_slots    */
#define MOE_ERR_TIMEOUT (-7)  /* a bounded device-side wait expired             */
#define MOE_ERR_STATIC (-8)   /* size beyond moe_route_static's fixed scratch    */

#define MOE_SLOT_REMOTE (-2)  /* slot-table entry: the expert lives on another GPU
                                 (expert parallelism): it contributes zero to this
                                 GPU's partial sums and is not an error            */

#define MOE_MAX_E 512         /* experts per layer                              */
#define MOE_MAX_TOPK 32
#define MOE_DECODE_MAX_T 8    /* decode path: a verify window of 1 + 4 drafts fits */
#define MOE_ROUTER_F64_MAX_T 128 /* chunks of up to this many tokens route with fp64
                                    tensor-core logits; longer ones with bf16 planes */
#define MOE_PREFILL_MAX_T 8192 /* one prefill chunk                             */

/*
 * Expert-slot layout, identical for every slot of an arena.  Matrix m is
 * 0 = gate [I, H], 1 = up [I, H], 2 = down [H, I], row-major by output row;
 * quant blocks of `block` (= 32) elements run along the reduction axis.
 * Codes: row r of a b-bit matrix with reduction length K occupies K*b/8
 * bytes at off_codes[m] + r*K*b/8; element c sits at byte c*b/8 of the row,
 * bit offset (c*b) % 8, least significant bits first.  Scales: fp16
 * [rows][K/32] at off_scales[m].  Slot s starts at arena + s*slot_bytes.
 * Requirements (else MOE_ERR_SHAPE): block == 32, H % 32 == 0, I % 32 == 0,
 * 32 <= H <= 8192, 32 <= I <= 4096, bits in {2, 4}, slot_bytes % 256 == 0,
 * every offset % 128 == 0 with its section inside the slot, n_slots >= 1,
 * reserved == 0.  The prefill path also needs H % 128 == 0 and I % 128 == 0.
 */
typedef struct moe_arena_desc {
    int32_t H, I, block;
    int32_t bits_gate, bits_up, bits_down;
    int64_t slot_bytes;
    int64_t off_codes[3];
    int64_t off_scales[3];
    int32_t n_slots;
    int32_t reserved;        /* must be 0 */
} moe_arena_desc;

/*
 * Optional routing outputs of a forward call.  Each non-NULL pointer is a
 * device buffer the call fills (it is also used as the working copy, so
 * passing it costs no extra traffic):
 *   topk_idx [T*top_k] int32  experts of token t in slots j = 0..k-1,
 *                             ordered by logit desc, ties by lower index
 *   topk_w   [T*top_k] fp32   gate weights (softmax over the k chosen logits)
 *   expert_offsets [E+1]      exclusive prefix sum of per-expert pair counts
 *   perm     [T*top_k] int32  pair ids p = t*k + j grouped by expert,
 *                             ascending p inside an expert
 *   n_rechecked [1] int32     tokens whose selection needed the exact fp64
 *                             re-evaluation (diagnostic)
 */
typedef struct moe_route_out {
    int32_t* topk_idx;
    float* topk_w;
    int32_t* expert_offsets;
    int32_t* perm;
    int32_t* n_rechecked;
} moe_route_out;

/* Bytes of scratch workspace a forward (or moe_route) call with these sizes
 * needs; pass it as `ws` (device, 256-byte aligned).  Non-decreasing in T: a
 * workspace sized for T serves every call with at most T tokens and the same
 * E, top_k, H and I.  Host only, no CUDA. */
size_t moe_workspace_bytes(int T, int E, int top_k, int H, int I);

/*
 * Router and grouping only.  Defined by the "Strata Coder deep-dive" page,
 * section 1 (each token of a layer is routed to 10 of its 512 experts, 256 in
 * the pruned variant of section 2), and the "Coder benchmark record" page,
 * "why Coder is fast" (experts addressed and fetched per (layer, expert)):
 * logits l = x W_r^T + b, the top_k experts by (l desc, e asc) - bit-exact
 * against the fp64 sequential definition, certified on the device - their
 * softmax gate weights, and the pairs (t, j) grouped by expert.  The logits
 * that the certification starts from are fp64 with per-entry bounds for
 * T <= MOE_DECODE_MAX_T, fp64 from the fp64 tensor cores for
 * T <= MOE_ROUTER_F64_MAX_T, and fp32 sums of exact bf16 planes on the
 * tensor cores above (E % 128 == 0, H % 64 == 0; other shapes: CUDA cores).
 *   x [T][H] bf16 (device, 16-B aligned), router_w [E][H] fp32 (device,
 *   16-B aligned), router_bias [E] fp32 (device) or NULL.
 *   Outputs (device): topk_idx [T*k], topk_w [T*k], expert_offsets [E+1],
 *   perm [T*k].  1 <= T <= 8192, 1 <= E <= 512, 1 <= top_k <= min(E, 32).
 *   T = 0 is a no-op returning MOE_OK.
 */
int moe_route(const uint16_t* x, int T, int H, const float* router_w, const float* router_bias,
              int E, int top_k, int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
              int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_route without a caller workspace: the same router and grouping kernels,
 * with their scratch in a fixed device array inside libmoe.so
 * (MOE_ROUTE_STATIC_BYTES per device; every GPU that loads the library holds
 * it until the process exits).  No page of the method has a counterpart: it
 * is a serving convenience for callers that cannot hand over a workspace, and
 * it allocates nothing (no cudaMalloc, no cudaFree, no allocator of any kind).
 * The array's device address is looked up with cudaGetSymbolAddress by the
 * first call in each CUDA context of a device (again after cudaDeviceReset or
 * under another context); make that first call before any stream capture.
 *   Arguments, layouts and outputs as moe_route.  Limits: 1 <= T <=
 *   MOE_ROUTE_STATIC_MAX_T, 1 <= E <= 512, 1 <= top_k <= min(E, 32); a T
 *   above the limit returns MOE_ERR_STATIC before any CUDA call.  T = 0 is a
 *   no-op returning MOE_OK.  The rechecked-candidate counter in the scratch
 *   is cleared on the stream at every call; everything else is overwritten.
 *   Concurrency: every call on a device shares the one scratch array, so two
 *   calls whose kernels overlap on the GPU (different streams, or different
 *   host threads without ordering) race and may return wrong routes.  Order
 *   them on one stream.
 */
#define MOE_ROUTE_STATIC_MAX_T 8
#define MOE_ROUTE_STATIC_BYTES (128 * 1024)
int moe_route_static(const uint16_t* x, int T, int H, const float* router_w, const float* router_bias,
                     int E, int top_k, int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                     int32_t* perm, void* stream);

/*
 * Full layer for a decode window, 1 <= T <= MOE_DECODE_MAX_T: router, grouping,
 * fused dequant + SwiGLU gate/up, down projection, weighted combine (+x when
 * residual != 0) and, when hist != NULL, hist[layer][e] += pairs routed to e.
 * Defined by the "Strata Coder deep-dive" page, sections 1-3 (10 of 512
 * experts per token; an expert is gate, up and down projections stored
 * block-quantized at low bit width, gate/up narrower than down) and the
 * "Coder benchmark record" page, test environment (a verify window of the
 * token plus 4 speculative drafts, T = 5) and "why Coder is fast" (each
 * selected expert's weights are read once per window).
 *   desc (host); arena (device, 256-B aligned); slot_table [L][E] int32
 *   (device); x [T][H] bf16 (device); out [T][H] bf16 (device);
 *   steer [H] fp32 (device, 16-B aligned) or NULL: the steering projection of
 *   the "Coder benchmark record" page (steering vector section) - each output
 *   row h (residual included) becomes h - (h . v) v before its one bf16
 *   rounding, v = steer used as given (a unit vector is the caller's
 *   business); NULL = no projection;
 *   hist [L][E] uint32 (device, persistent, caller-owned) or NULL;
 *   route_out (host struct of device pointers) or NULL.
 *   0 <= layer < L.  T = 0 is a no-op.
 */
int moe_forward_decode(const moe_arena_desc* desc, const void* arena, const int32_t* slot_table,
                       int L, int layer, const uint16_t* x, int T, const float* router_w,
                       const float* router_bias, int E, int top_k, int residual, const float* steer,
                       uint16_t* out, uint32_t* hist, const moe_route_out* route_out, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * Full layer for a prefill chunk, 1 <= T <= MOE_PREFILL_MAX_T: same arguments
 * and results as moe_forward_decode; the expert FFN runs as per-expert grouped
 * GEMMs on the tensor cores (weights dequantised to bf16 on chip, SwiGLU
 * output h rounded to bf16, per-pair expert outputs kept in bf16).  Defined
 * by the same passages as moe_forward_decode, with the chunked prompt path of
 * the "Coder benchmark record" page, test environment (prompts processed in
 * chunks of at most 8,192 tokens), and of the "Strata overview" page, chunked
 * prefill.
 */
int moe_forward_prefill(const moe_arena_desc* desc, const void* arena, const int32_t* slot_table,
                        int L, int layer, const uint16_t* x, int T, const float* router_w,
                        const float* router_bias, int E, int top_k, int residual, const float* steer,
                        uint16_t* out, uint32_t* hist, const moe_route_out* route_out, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * Routing-count histogram ("--dump-routing" counts of the benchmark record
 * page): hist[layer][e] += expert_offsets[e+1] - expert_offsets[e] for
 * e < E, one owner thread per expert, no atomics.  expert_offsets [E+1]
 * (device), hist [L][E] uint32 (device).  The update is a plain read-add-
 * write: calls (and forward calls with hist != NULL) that add to the same
 * hist must be ordered, e.g. on one stream; concurrent ones lose counts.
 */
/*
 * Expert parallelism: experts e mod G on G GPUs, the router replicated, an
 * all-gather of x and a reduce-scatter of fp32 partial outputs (the "Picking
 * a quant" page's multi-GPU section gives splitting a model over GPUs as
 * prior art; the layer's arithmetic is moe_forward_decode's).  Each GPU calls moe_forward_partial on the
 * gathered tokens with a slot table in which the experts it does not hold are
 * MOE_SLOT_REMOTE; the caller sums the G partials (a reduce-scatter) and
 * moe_finish_rows adds the residual and rounds.
 *
 * moe_forward_partial: the same arguments as moe_forward_decode (prefill != 0:
 * as moe_forward_prefill) except that there is no residual, no steering and
 * no bf16 output: partial [T][H] fp32 (device, 16-B aligned) receives, per
 * token, the gate-weighted sum of its selected experts' outputs over the
 * experts whose slot is held here, in slot order (the combine of the
 * forwards before its residual and its rounding).  The routing (and
 * route_out, hist) covers all k selections of every token, remote ones
 * included, so every GPU sees the same routing.  Errors as the forwards.
 */
int moe_forward_partial(int prefill, const moe_arena_desc* desc, const void* arena, const int32_t* slot_table,
                        int L, int layer, const uint16_t* x, int T, const float* router_w,
                        const float* router_bias, int E, int top_k, float* partial, uint32_t* hist,
                        const moe_route_out* route_out, void* ws, size_t ws_bytes, void* stream);

/*
 * out[t][c] = bf16((residual ? x[t][c] : 0) + sum[t][c]) for T rows of H,
 * with the steering projection applied first when steer != NULL (as in the
 * forwards: r - (r . v) v on the fp32 row, residual included).  x [T][H] bf16,
 * sum [T][H] fp32, steer [H] fp32 or NULL, out [T][H] bf16, all device,
 * 16-B aligned; H % 8 == 0.  The finishing step of an expert-parallel layer
 * (the combine's last two steps of the "Coder benchmark record" page's layer:
 * residual add and one rounding; steering as its steering vector section).
 */
int moe_finish_rows(const uint16_t* x, const float* sum, int T, int H, int residual, const float* steer,
                    uint16_t* out, void* stream);

int moe_route_histogram(const int32_t* expert_offsets, int E, int L, int layer, uint32_t* hist,
                        void* stream);

/*
 * Expert-profile ranking (Strata Coder deep-dive page, section 3; benchmark
 * record page, "expert profile file"): every (layer, expert) pair ordered by
 * count descending, ties by (layer, expert) ascending.
 *   hist_host [L][E] uint32 (host); pairs_out [L*E][2] uint16 (host) =
 *   (layer, expert) of rank 0, 1, ...  Host only, no CUDA.
 */
int moe_rank_experts(const uint32_t* hist_host, int L, int E, uint16_t* pairs_out);

/*
 * Expert profile file in the STRP v1 layout of the "Coder benchmark record"
 * page, "expert profile file": the magic "STRP", a header of five uint32
 * (version = 1, layers L, experts per layer E, ranked pairs n, inverse-table
 * entries = L*E), the n ranked (layer, expert) pairs as two uint16 each in
 * rank order, then one inverse table per layer of E int32 entries giving the
 * rank of (layer, expert), -1 = unranked (O(1) lookup of a pair's place).
 * All fields little-endian.  The page lists the header fields without
 * saying which of its two counts is which; here "ranked pairs" counts the
 * body and "entries" the inverse tables.  Host only, no CUDA.
 * moe_profile_bytes: the file size for (n_pairs, L, E), -1 if out of range
 *   (1 <= L, E <= 65535, 0 <= n_pairs <= L*E).
 * moe_profile_write: pairs [n_pairs][2] uint16 (host) = (layer, expert) in
 *   rank order, e.g. a prefix of moe_rank_experts' output; writes the file
 *   into buf (host, buf_bytes) and returns its size, or the size alone when
 *   buf == NULL; MOE_ERR_ARG for a pair out of range or ranked twice,
 *   MOE_ERR_WS when buf is too small, MOE_ERR_RANGE for bad sizes.
 * moe_profile_read: parses and validates a file; fills L, E, n_pairs and,
 *   when not NULL, pairs [n_pairs][2] and inverse [L*E]; MOE_ERR_SHAPE for a
 *   malformed file.
 * moe_profile_hit_rate: the slot-budget simulator of the same page ("why a
 *   72% hit rate proves the mapping"): with the first `slots` ranked pairs
 *   resident, the fraction of the routed reads counted in hist [L][E] (host,
 *   e.g. a routing histogram of a held-out run) that land on a resident pair;
 *   -1 on bad arguments.
 */
int64_t moe_profile_bytes(int n_pairs, int L, int E);
int64_t moe_profile_write(const uint16_t* pairs, int n_pairs, int L, int E, uint8_t* buf, size_t buf_bytes);
int moe_profile_read(const uint8_t* buf, size_t bytes, int* L, int* E, int* n_pairs, uint16_t* pairs,
                     int32_t* inverse);
double moe_profile_hit_rate(const uint16_t* pairs, int n_pairs, int L, int E, int slots, const uint32_t* hist);

/* Reads and clears the current device's status word after synchronising
 * `stream`: MOE_OK, MOE_ERR_SLOT or MOE_ERR_TIMEOUT (the first latched), or
 * MOE_ERR_RANGE if an internal index was out of range and replaced (a
 * library fault; inputs cannot cause it: non-finite logits rank as -inf).
 * No page defines it: it is the boundary's way of reporting what the device
 * detects without trapping. */
int moe_last_device_error(void* stream);

/* Static message for a return code (the boundary's error contract; no page
 * defines it).  Never NULL: an unknown code gets a generic message. */
const char* moe_strerror(int code);

/*
 * Measurement hooks (no counterpart on the source pages; used by the
 * benchmark).  moe_set_stage_events(events, n): when n >= 5, every later
 * forward call records the caller's CUDA events (cudaEvent_t, created with
 * timing enabled) on its stream at the stage boundaries: events[0] before the
 * router, [1] after grouping, [2] after the first expert stage (gate/up),
 * [3] after the second (down), [4] after the combine; a call that runs as
 * one fused kernel records only [0] before it and [1] after it (each record
 * in a graph costs microseconds of device time).  n = 0 (or events = NULL)
 * turns it off.  The setting is process-wide and read at call time, so
 * a call captured into a CUDA graph records into the events set at capture.
 * moe_launch_count(): kernels this process has launched through the library
 * (host-side counter; launches replayed from a captured graph are not added).
 */
int moe_set_stage_events(void* const* events, int n);
uint64_t moe_launch_count(void);

/*
 * Test hooks (no counterpart on the source pages; off by default, never used
 * by the layer itself):
 * moe_debug_set(MOE_DBG_SPIN_LIMIT, n): grid-barrier waits of the fused decode
 *   kernel give up after n polls instead of about 2 s worth (0 restores it).
 * moe_debug_set(MOE_DBG_BARRIER_EXTRA, n): the fused decode kernel's first
 *   grid barrier waits for n arrivals that never come, so that every CTA
 *   runs into the polling bound and reports MOE_ERR_TIMEOUT (site 1) with no
 *   copy in flight and no tensor memory held; 0 restores it.
 * Both are process-wide and read when a forward call is enqueued.
 * moe_workspace_offset(T, E, top_k, H, I, field): byte offset inside a forward
 *   or route workspace of MOE_WS_FAST_LOGITS (the router's fast logits: fp32
 *   [T][E] for chunks T > MOE_ROUTER_F64_MAX_T, fp64 for shorter ones) or
 *   MOE_WS_PAIR_OUT (per-pair expert outputs w * y in pair order: bf16 [T*k][H]
 *   for chunks) or MOE_WS_SLOW_COUNT (int32: how many tokens of a chunk the
 *   fast certification could not decide, then their ids); (size_t)-1 for bad
 *   arguments.
 * moe_router_gamma(T, E, H): for a chunk (T > MOE_DECODE_MAX_T), the factor
 *   gamma of the fast logits' certified bound |fast - exact| <= gamma *
 *   (||x_t|| ||W_r[e]|| + |b_e|) (before the fp64 definition's own rounding
 *   term); -1 for decode windows or bad sizes.
 */
#define MOE_DBG_SPIN_LIMIT 1
#define MOE_DBG_BARRIER_EXTRA 2
#define MOE_WS_FAST_LOGITS 1
#define MOE_WS_PAIR_OUT 2
#define MOE_WS_SLOW_COUNT 3
int moe_debug_set(int key, int value);
size_t moe_workspace_offset(int T, int E, int top_k, int H, int I, int field);
double moe_router_gamma(int T, int E, int H);

/* Diagnostic companion of MOE_ERR_TIMEOUT: after synchronising `stream`,
 * returns and clears where the first bounded device wait gave up
 * (site * 1000000 + CTA * 1000 + unit, 0 = none); negative on CUDA failure. */
int moe_timeout_site(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
