/*
 * moe_sparse.h -- C ABI of the routed-expert MoE layer with intra-expert
 * activation sparsity, for NVIDIA B200 (sm_100a).
 *
 * The operation ("Uncovering Intra-expert Activation Sparsity for Efficient
 * Mixture-of-Expert Model Execution", technical summary, Methodology item 3;
 * Hindi summary of the same paper, "How they did it: the skip-list system"):
 * per token x (d_model values),
 *
 *   router     p = softmax(x Wr^T) over all E experts; the top_k experts by p
 *              are selected (ties go to the lower index); weight w_e = p_e
 *              (the router is kept unchanged; no renormalisation).
 *   gate       g = x Wg[e]                      dense, every neuron of e
 *   mask       neuron j active iff |silu(g_j)| >= tau    one pass, no sort
 *   up/down    y += w_e * sum_{j active} silu(g_j) (x Wu[e][:,j]) Wd[e][j][:]
 *   shared     y += sum_j silu(x Ws_g[:,j]) (x Ws_u[:,j]) Ws_d[j][:]
 *              for each shared expert, every neuron, unweighted.
 *   out        bf16(y), round to nearest even.
 *
 * Conventions for every function:
 *   - bf16 tensors are passed as raw 16-bit patterns (any bf16 type works).
 *   - "device pointer" means memory of the current CUDA device, "host
 *     pointer" ordinary (pageable or pinned) host memory.
 *   - `stream` is a cudaStream_t cast to void* (NULL = the legacy default
 *     stream).  All work is enqueued on it; calls return once it is enqueued
 *     unless stated otherwise.
 *   - Every function returns MOE_OK (0) or a negative MOE_E* code; argument
 *     errors are detected on the host before anything is launched.  No C++
 *     exception crosses this boundary.
 *   - A handle must only be used from one host thread at a time and only on
 *     the device that was current when it was created.
 */
#ifndef MOE_SPARSE_H
#define MOE_SPARSE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_EINVAL (-1)   /* bad size, NULL pointer, NaN tau, ...            */
#define MOE_ENOMEM (-2)   /* device or host allocation failed (create only)  */
#define MOE_ECUDA (-3)    /* a CUDA runtime call or kernel launch failed     */
#define MOE_EALIGN (-4)   /* a pointer is not 16-byte aligned                */
#define MOE_EHANDLE (-5)  /* NULL or destroyed handle                        */
#define MOE_EDEVICE (-6)  /* a kernel reported an error (e.g. a bounded wait
                             ran out); read by moe_query_stats.  The forward
                             in which it happened produced wrong output;
                             later forwards start with a clear error state
                             and are unaffected                              */
#define MOE_ENOTSUP (-7)  /* shape or path not supported by this build       */

/* Path selection (moe_set_path). */
#define MOE_PATH_AUTO 0    /* sparse gather path for T <= T*, dense above   */
#define MOE_PATH_SPARSE 1  /* always the sparse gather path                 */
#define MOE_PATH_DENSE 2   /* always the tensor-core grouped GEMM, masked    */

typedef struct moe_sparse_s *moe_handle;

/* Layer weights, all DEVICE pointers to bf16, caller-owned, x @ W layout:
 *   w_router [E][d_model]
 *   w_gate   [E][d_model][d_ff]      w_up [E][d_model][d_ff]
 *   w_down   [E][d_ff][d_model]
 *   ws_gate, ws_up [n_shared][d_model][d_ff], ws_down [n_shared][d_ff][d_model]
 *   (ws_* must be NULL when n_shared == 0; the shared d_ff equals d_ff).
 * Every pointer must be 16-byte aligned. */
typedef struct {
    const void *w_router;
    const void *w_gate;
    const void *w_up;
    const void *w_down;
    const void *ws_gate;
    const void *ws_up;
    const void *ws_down;
} moe_weights;

/* Statistics of the last forward on a handle (moe_query_stats). */
typedef struct {
    int path;              /* MOE_PATH_SPARSE or MOE_PATH_DENSE                 */
    int n_tokens;          /* T                                                  */
    int n_touched;         /* distinct routed experts selected by the batch      */
    int t_star;            /* current sparse/dense switch point                  */
    long long n_active;    /* sum over (token, expert) pairs of active neurons   */
    long long n_union;     /* sum over touched experts of the union of their
                              tokens' active neurons (rows of Wu/Wd read)        */
    double alg_bytes;      /* algorithmic HBM bytes of the sparse path:
                              full Wg of touched experts + 2*d_model*2 bytes per
                              union-active neuron + shared experts + router +
                              x and out                                          */
    double dense_bytes;    /* the same for the dense path (all neurons)          */
    int device_error;      /* first device error code since the previous
                              moe_query_stats (0: none)                          */
    int fused_router;      /* the last forward's moe_set_fused_router mode if it
                              routed the batch inside the expert kernel (1: no
                              router launch, 2: one launch), else 0              */
    int capacity;          /* pairs per expert the last forward kept at most
                              (moe_set_capacity), -1 if it dropped none          */
    int deterministic;     /* the last forward combined in a fixed order
                              (moe_set_deterministic)                            */
} moe_stats;

/* Create a layer.  Copies and repacks the weights into library-owned device
 * memory (the caller may free its tensors afterwards) and allocates all
 * workspace for up to `max_tokens` tokens per call, so that forward calls
 * never allocate.  Synchronises the device before returning.
 * Requirements (else MOE_EINVAL): 1 <= top_k <= E <= 1024; 8 <= d_model <= 4096
 * and d_model % 8 == 0 (eight gate rows must sit in at most two 32 KB stages); d_ff >= 32 and d_ff % 32 == 0; d_ff <= 65535;
 * 0 <= n_shared <= 8; 1 <= max_tokens <= 65536 (0 selects 4096).
 * Pointers must be 16-byte aligned (else MOE_EALIGN).  On failure *out is
 * set to NULL and nothing is leaked. */
int moe_sparse_create(const moe_weights *w, int E, int top_k, int d_model, int d_ff,
                      int n_shared, int max_tokens, moe_handle *out);

/* The masked layer.  x: DEVICE [T][d_model] bf16; out: DEVICE [T][d_model]
 * bf16 (may not alias x).  1 <= T <= max_tokens.  tau <= 0 keeps every
 * neuron, tau = +inf keeps none; NaN tau is MOE_EINVAL.  The path follows
 * moe_set_path (AUTO by default: sparse for T <= T*, the dense masked GEMM
 * above).  Both paths give the same layer up to rounding.  Asynchronous. */
int moe_sparse_forward(moe_handle h, const void *x, int T, float tau, void *out, void *stream);

/* The unmasked layer (every neuron active) on the dense tensor-core path:
 * the baseline the sparse path is measured against.  Same arguments and
 * rules as moe_sparse_forward without tau. */
int moe_dense_forward(moe_handle h, const void *x, int T, void *out, void *stream);

/* Same as moe_sparse_forward but x and out are HOST pointers: copies x in,
 * runs the layer and copies out back on `stream`, then synchronises it. */
int moe_sparse_forward_host(moe_handle h, const void *x_host, int T, float tau, void *out_host,
                            void *stream);

/* Free everything the handle owns (synchronises the device first).  NULL is
 * ignored; the handle must not be used afterwards. */
void moe_sparse_destroy(moe_handle h);

/* Force a path (MOE_PATH_*) for subsequent forwards; MOE_EINVAL otherwise. */
int moe_set_path(moe_handle h, int path);

/* Set the switch point T* of MOE_PATH_AUTO (sparse iff T <= t_star). */
int moe_set_t_star(moe_handle h, int t_star);

/* Measure the switch point of MOE_PATH_AUTO on this device for this layer:
 * for batch sizes 1, 2, 3, 4, 6, 8, 12, 16, 24, ... up to T_max, the first T
 * rows of x (DEVICE [T_max][d_model] bf16, a representative batch) run through
 * both branches at threshold tau (the sparse branch's cost depends on it),
 * each captured into a CUDA graph on a private stream and timed on the
 * device as one graph launch (median of five; before every run a 2 x L2
 * buffer is written and read back, so L2 holds no useful and no dirty line),
 * so neither branch is charged for host gaps between its kernels; the
 * sparse time is the mean over two disjoint batches of T rows (the first
 * and the last T rows of x) where T_max >= 2T, since the sparse branch's
 * cost varies with how a batch routes; the search stops at the first T whose
 * sparse time exceeds 95 % of the dense one, and T* becomes the last T
 * before it; it is stored in the handle and
 * in *t_star_out (HOST pointer).
 * ("Uncovering Intra-expert Activation Sparsity...", technical summary,
 * Methodology item 3, "Dynamic switching": sparse for small batches, dense
 * for large.)  Allocates and frees a 2 x L2-sized flush buffer; synchronises
 * `stream`; the launch events of moe_set_launch_events are not recorded
 * meanwhile.  Without a dense branch T* becomes INT_MAX.  Until this is
 * called, T* is 16 (measured on the OLMoE-shaped layer at 90% sparsity). */
int moe_tune_t_star(moe_handle h, const void *x, int T_max, float tau, int *t_star_out, void *stream);

/* Decode batches on the sparse path (T within one token tile of the expert
 * kernel: up to 16 tokens for d_model <= 2048, up to 8 above; T * top_k <= 128,
 * T * E <= 8192, d_model >= 64) normally route inside the expert kernel: each
 * CTA computes some experts' logits, all CTAs then select the top-k and build
 * the plan themselves, so no router kernel and no plan hand-off precede the
 * gate stream.  mode = 0 uses the separate router kernel instead (same
 * results up to the order of fp32 sums in the logits); 1 restores the
 * default (two launches: the expert kernel, then a small kernel converting
 * the fp32 accumulator to the bf16 output); 2 also does that conversion at
 * the end of the expert kernel, after a grid-wide count of the CTAs whose
 * sums have landed, so such a forward is one launch (router, gate, mask,
 * gather, up/down and combine; measured 2.5-3 us slower than mode 1 at
 * 1 and 16 tokens on B200, which is why it is not the default).  Modes 1
 * and 2 assume every CTA of the expert kernel (at most one per SM) can be
 * resident at once, which holds unless the context is restricted to fewer
 * SMs than the device has; otherwise the routing wait runs out and reports
 * error code 55 (57 for the combine's count).  Other modes: MOE_EINVAL. */
int moe_set_fused_router(moe_handle h, int mode);

/* Router only: idx_out [T][top_k] int32 and w_out [T][top_k] fp32, both
 * DEVICE pointers, in rank order.  Asynchronous. */
int moe_debug_router(moe_handle h, const void *x, int T, int *idx_out, float *w_out, void *stream);

/* Runs the sparse path and writes each (token, rank) pair's active-neuron
 * list: idx_out DEVICE [T][top_k][d_ff] uint16, ascending, the first
 * cnt_out[t][r] entries valid; cnt_out DEVICE [T][top_k] int32.  out may be
 * NULL (the layer output is then discarded).  Asynchronous. */
int moe_debug_active(moe_handle h, const void *x, int T, float tau, uint16_t *idx_out,
                     int *cnt_out, void *out, void *stream);

/* Threshold for a target sparsity q in [0, 1]: runs the router and the gate
 * projection for x (DEVICE [T][d_model] bf16) and stores in *tau_out (HOST
 * pointer) the floor(q*N)-th smallest score |silu(g)| (0-based, exact
 * selection) among the N = T*top_k*d_ff scores of the (token, expert) pairs the
 * router selects; shared experts are excluded.  q <= 0 gives 0 and
 * floor(q*N) >= N gives +inf.  About 1 - q of the routed neurons then have
 * s >= tau ("Uncovering Intra-expert Activation Sparsity...", Results:
 * per-model sparsity cutoffs are set as a fraction of neurons kept).
 * The first call allocates a score buffer of max_tokens*max(top_k, n_shared)*d_ff
 * floats that the handle keeps (MOE_ENOMEM if that fails).  Synchronises
 * `stream`. */
int moe_calibrate_tau(moe_handle h, const void *x, int T, double sparsity, float *tau_out,
                      void *stream);

/* The shared experts' own threshold ("Uncovering Intra-expert Activation
 * Sparsity...", technical summary, Methodology item 1: shared-expert neurons
 * matter more per neuron than routed ones, so they take a separate, looser
 * threshold).  On later masked forwards (moe_sparse_forward, either path) a
 * shared neuron j counts iff |silu(x Ws_g[:,j])| >= tau_shared; tau_shared
 * <= 0 (the default) keeps every shared neuron, +inf none.  moe_dense_forward
 * stays unmasked.  NaN is MOE_EINVAL.  moe_query_stats' byte counts still
 * count the shared experts in full. */
int moe_set_shared_tau(moe_handle h, float tau_shared);

/* A per-pair rank budget in place of the routed threshold ("Uncovering
 * Intra-expert Activation Sparsity...", technical summary, Methodology item
 * 1: the lowest-scoring neurons of an expert are zeroed progressively).  With
 * r >= 0, later masked forwards (moe_sparse_forward, moe_debug_active) keep,
 * for every routed (token, expert) pair, the r neurons with the largest
 * s = |silu(g)| (fp32); equal scores go to the lower neuron index, a NaN score
 * is never kept, so a pair keeps min(r, its non-NaN scores) neurons; `tau`
 * is then unused for the routed experts, and the shared experts keep their
 * moe_set_shared_tau rule.  r < 0 returns to the threshold (the default).
 * The selection is exact and sort-free (a radix select of each pair's f
 * scores).  The budget runs on the sparse path at every batch size: a forward
 * forced onto the dense path (moe_set_path) returns MOE_ENOTSUP.  It costs
 * two sparse passes (the routed gates, then the masked up/down reading the
 * gates back) and one small selection kernel in between.  The first call with
 * r >= 0 allocates max_tokens * top_k * (d_ff + 2) floats (MOE_ENOMEM if that
 * fails, the setting unchanged); moe_sparse_destroy frees them. */
int moe_set_rank_budget(moe_handle h, int r);

/* Capacity-aware token drop ("Capacity-Aware Inference" page, section
 * "Capacity-Aware Token Drop"): with gamma > 0, on later forwards every
 * routed expert holds at most C = ceil(gamma * T * top_k / E) of the batch's
 * (token, expert) pairs (the mean load times the capacity factor, rounded
 * up).  An expert routed more pairs keeps the C with the largest routing
 * weight (softmax probability, fp32), equal weights going to the lower token
 * index; the dropped pairs contribute nothing (their mask lists are empty),
 * the kept ones keep their weights (no renormalisation), and the shared
 * experts are unaffected.  moe_debug_router still reports the router's
 * selection before the drop; moe_query_stats' counts are after it.  The drop
 * is applied in the router kernel's bucketing, so such forwards do not route
 * inside the expert kernel; a batch of more than 4096 pairs whose capacity is
 * below T returns MOE_ENOTSUP (C >= T drops nothing and is always allowed).
 * gamma <= 0 (the default) turns it off; NaN is MOE_EINVAL.  The dropping
 * makes pairs' work depend on the rest of the batch, which is the method's
 * intent; outputs then differ from the plain layer. */
int moe_set_capacity(moe_handle h, float gamma);

/* Deterministic combine ("Uncovering Intra-expert Activation Sparsity ...",
 * technical summary, Methodology item 3: the routed experts' outputs are
 * weighted and summed into the token's output, plus the shared experts').
 * By default every contribution is added into an fp32 accumulator with
 * atomics, so the rounding of that sum follows the order in which the
 * hardware lands them and a repeated forward can differ in the last bf16
 * bit.  With enable != 0, later forwards (both paths, every launch mode)
 * write each contribution -- one per (token, routing slot or shared expert,
 * 128-neuron block) on the sparse path, per (token, slot) on the dense one --
 * to a row of its own with plain stores, and the conversion adds a token's
 * rows in one fixed order: identical inputs then give bit-identical outputs,
 * whatever the schedule.  The cost is the rows' traffic: the sparse path
 * writes and reads back T * (top_k + n_shared) * ceil(d_ff / 128) * d_model
 * floats (8 MiB at 16 tokens of a 64-expert top-8 layer with d_model 2048 and
 * d_ff 1024).  The first call with enable != 0 allocates max_tokens *
 * (top_k + n_shared) * ceil(d_ff / 128) * d_model floats (MOE_ENOMEM if that
 * fails, the setting unchanged) and clears them; moe_sparse_destroy frees
 * them.  With it on, no row has two writers, so an item is never split
 * across CTAs by its records (on layers whose shared experts run without a
 * threshold those items are then the slowest of a decode step).  Not
 * stream-ordered: call it between forwards, with none in flight. */
int moe_set_deterministic(moe_handle h, int enable);

/* As moe_calibrate_tau, over the N = T*n_shared*d_ff scores of the shared
 * experts' neurons: the floor(q*N)-th smallest |silu(x Ws_g)| (0-based, exact
 * selection); q <= 0 gives 0 and floor(q*N) >= N gives +inf.  MOE_EINVAL when
 * the layer has no shared expert.  Shares the score buffer of
 * moe_calibrate_tau (allocated by the first of the two calls).  Synchronises
 * `stream`. */
int moe_calibrate_tau_shared(moe_handle h, const void *x, int T, double sparsity, float *tau_out,
                             void *stream);

/* Timing hook for benchmarks: on every later forward, record caller-owned CUDA
 * events (cudaEvent_t cast to void*, created on the handle's device) on the
 * forward's stream -- events[0] before the router kernel, events[1] between
 * the router and the expert kernel(s), events[2] after them; when the batch
 * is routed inside the expert kernel, events[1] directly follows events[0].
 * They are recorded with cudaEventRecordExternal, so a forward captured into
 * a CUDA graph records them on every replay.  n must be 3; events == NULL or
 * n == 0 stops recording.  The handle keeps the three handles, not the array. */
int moe_set_launch_events(moe_handle h, void *const *events, int n);

/* Tracing hook: when buf (DEVICE, 8-byte aligned, `bytes` long) is set, later
 * forwards stamp the GPU global timer (ns) at phase boundaries of each CTA.
 * The sparse path then runs a separately compiled, traced copy of its expert
 * kernel (same results; the stamps cost 4-7 % of a decode step, which the
 * untraced kernel does not pay).
 * The first half of the buffer holds 8 stamps per router CTA (CTA index
 * y*gridDim.x + x): start, logits done, top-k start, top-k done, plan start,
 * plan done (the last two only in the CTA that builds the plan).  The second
 * half holds 64 per expert-kernel CTA: [0] start, [1] plan loaded; for each
 * of the CTA's first three items i, at 2 + 10*i: metadata ready, gate
 * accumulator ready, mask read out (twice), mask step synchronised, mask and
 * lists published, first gathered batch in (up warps), first h in (down
 * warps), up projection done, down projection and flush done; the gate
 * lane's totals: [32] ns waiting to claim an item, [33] ns waiting for a free
 * ring stage, [34] stages issued, [35] issue time of the last stage; the up
 * warps' totals: [36] ns in mask steps, [37] ns waiting for the next item's
 * id and metadata slot; [40 + g] issue of gate stage g < 4; [44]..[47] routing
 * inside the kernel: start, own logits computed, logits staged, plan built;
 * [48 + q] token rows of
 * tile q < 4 ready (batches of more than 16 tokens; smaller batches stream
 * the token operand with the gate stages); [52], [53] the up warps' total
 * time waiting for and
 * working on gathered batches, [54], [55] the same for the down warps (ns);
 * [56], [57] first gate stage consumed and accumulator committed for item 0;
 * [58], [59], [60] routing inside the kernel: this CTA's logits published,
 * every expert's logits available, top-k selected;
 * [61] gathered records processed; [62] end; [63] the CTA's item count.
 * Unwritten slots keep their old contents.
 * buf == NULL turns tracing off. */
int moe_set_trace(moe_handle h, void *buf, long long bytes);

/* Statistics of the last forward.  Synchronises the stream of that forward
 * (which must still exist; after moe_tune_t_star, the stream passed to it)
 * and reads device counters back; not for timed loops.
 * Device errors: forward calls do not synchronise, so they cannot report
 * what their kernels find (a bounded wait that ran out, error codes >= 30).
 * Each forward starts with a clear error state, so an error affects only the
 * forward it happened in (whose output is then wrong).  This call reports
 * the FIRST device error code since its previous call in st->device_error,
 * returns MOE_EDEVICE for it, and clears it; 0 / MOE_OK when there was none. */
int moe_query_stats(moe_handle h, moe_stats *st);

/* Test-only fault injection (no GPU fault, trap or hang is involved).
 * MOE_INJECT_WITHHOLD_ITEMS: in the next sparse-path forward the expert
 * kernel's gate lane publishes no work item and issues no copy, so the other
 * agents' bounded waits for work run out (after about 10 ms); the kernel
 * records error code 50 and returns, that forward's output is wrong (zero),
 * and moe_query_stats then returns MOE_EDEVICE.  Applies once.
 * MOE_INJECT_NONE cancels a pending injection.
 * Separately, when the environment variable MOE_INJECT_ALLOC_FAIL is
 * "weights" or "workspace", moe_sparse_create treats that device allocation
 * as failed (MOE_ENOMEM, nothing leaked); "scores" does the same for the
 * first moe_calibrate_tau's score buffer, "rank" for the first
 * moe_set_rank_budget's buffers, "deterministic" for the first enabling
 * moe_set_deterministic's rows.
 * Device error codes of the sparse kernel: 30-36 (copy, MMA and token-tile
 * waits), 40-45 (the consumers' waits on accumulators, gathered records and
 * the hand-off of h), 50-54 (waits for work items, slots and claims), 55
 * (in-kernel routing: the other CTAs' logits), 56 (gate split: the other
 * parts' sums), 57 (the combine at the end: the other CTAs' flushes), 58
 * (gate split: the owner part's union list, which the other parts of the
 * item wait for to project their share of its records; every part is claimed
 * at kernel start, so this assumes all CTAs of the grid are resident, as the
 * in-kernel routing does). */
#define MOE_INJECT_NONE 0
#define MOE_INJECT_WITHHOLD_ITEMS 1
int moe_debug_inject(moe_handle h, int kind);

/* Size of the fixed device scratch used by moe_router_topk_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (4 << 20)

/* Router softmax top-k that allocates nothing, for callers that cannot call
 * cudaMalloc: servers that reserve all device memory up front in their own
 * arena, custom operators inside another framework that owns the allocator,
 * and latency-critical paths where an allocation's implicit synchronisation
 * is not acceptable.  The paper has no counterpart of this entry point; it
 * computes the same routing as the router step of moe_sparse_forward (softmax
 * over all E experts, top_k by probability, ties to the lower index, weight =
 * probability) without a handle:
 *   x        DEVICE [T][d_model] bf16, 16-byte aligned
 *   w_router DEVICE [E][d_model] bf16, 16-byte aligned
 *   idx_out  DEVICE [T][top_k] int32, w_out DEVICE [T][top_k] fp32, rank order
 * Its scratch (the T*E fp32 logits, rounded up to 256 bytes, plus one int per
 * 8 tokens) lives in a file-scope device array of MOE_NOALLOC_SCRATCH_BYTES
 * that every GPU loading the library keeps until the process exits; larger
 * T*E (or more than 65535 tiles of 8 tokens) is rejected with MOE_ENOTSUP
 * before anything is launched (e.g. E = 64 allows T up to 16352).  Other limits as moe_sparse_create: 1 <= top_k <= E
 * <= 1024, d_model % 8 == 0.  The first call on a device looks up the array's
 * device address with that device current, so make it before any stream
 * capture.  Under CUDA's lazy module loading (the default) that first call is
 * also when the library's device code and this array are loaded onto the
 * device, which needs MOE_NOALLOC_SCRATCH_BYTES plus the code of free device
 * memory: a caller whose own arena takes all device memory should make one
 * call at initialisation, before reserving it (or load modules eagerly with
 * CUDA_MODULE_LOADING=EAGER), after which calls need no free memory.  All calls share the array: calls that overlap on the GPU (on
 * different streams) race and must be serialised by the caller.  Each call
 * clears the tickets it needs with cudaMemsetAsync and calls no allocating
 * routine.  Asynchronous on `stream`. */
int moe_router_topk_noalloc(const void *x, int T, const void *w_router, int E, int d_model, int top_k,
                            int *idx_out, float *w_out, void *stream);

/* Static English text for an error code. */
const char *moe_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_SPARSE_H */
