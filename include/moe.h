/*
 * moe.h -- C ABI of the B200 routed-expert layer library (libmoe.so).
 *
 * The layer is the one the Edge0 streaming-MoE pages describe: an 8-bit router
 * with top-K softmax gating, routed experts stored as 4-bit affine group-64
 * matrices (SwiGLU gate/up/down), an unmerged LoRA delta, a shared expert
 * scaled by an 8-bit sigmoid gate, the weighted combine, and a Prerouter MLP
 * head predicting the next layer's top-K.  Sources: 2kiu.com article "iPhone,
 * Mac, Android, Windows measured: Edge0 on five platforms" (bullets "SSD expert
 * offload", "Prerouter", "Recover-LoRA"; paragraph on config.json: group_size
 * 64, bits 4, router gate and shared expert gate at 8 bits); autoark.ai Edge0
 * blog (tier table: 40 layers / 256 experts / K=4 and 24 / 128 / K=8);
 * news18a.com Edge0 article (Prerouter input = hidden state + executed experts;
 * prediction, expert I/O and LoRA delta as separate native components).
 *
 * Conventions shared by every call
 * --------------------------------
 * Ownership:  the caller allocates every device buffer (weights, activations,
 *             outputs, workspace).  The library allocates nothing and keeps no
 *             state between calls, apart from the allocation-free variant's
 *             fixed scratch array (moe_expert_forward_noalloc) and the looked-up
 *             address of the driver's tensor-map encoder.  All pointers are
 *             device pointers unless a
 *             comment says "host".  Structs are read on the host during the call
 *             and may be freed when it returns.
 * Asynchrony: work is enqueued on `stream` (a cudaStream_t passed as void*;
 *             NULL = legacy default stream).  A call returns after enqueueing.
 * Errors:     argument/shape checks run on the host before any launch and return
 *             MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE with
 *             nothing enqueued.  A failed launch returns MOE_ERR_CUDA.  What the
 *             device finds while the work runs is reported through an optional
 *             error word (err_word: one device int32, or NULL to ignore): a call
 *             stores a nonzero moe_status there if the slot still holds 0 (the
 *             first error wins) and never clears it, so one word can collect the
 *             status of many calls; read it after synchronising the stream.
 *             MOE_ERR_TIMEOUT: a device-side bounded wait gave up (the call's
 *             outputs are then undefined).  MOE_ERR_RANGE: an activation u is
 *             outside fp16's range (|u| > 65504); the kernels multiply bf16
 *             activations as fp16, which holds every bf16 value up to 65504
 *             exactly down to 2^-14 and rounds smaller ones (gradual underflow),
 *             so that row's outputs are undefined.
 * Determinism: results are bitwise reproducible for fixed inputs and launch
 *             shapes; no atomics accumulate into outputs.
 * Formats:    bf16/fp16 values are passed as their 16-bit patterns.
 *   Row record (one row of a quantised matrix with in_dim inputs, `bits` 4 or
 *     8): the codes (in_dim*bits/8 bytes; a 4-bit element k sits at bits
 *     4*(k%8) of little-endian 32-bit word k/8, an 8-bit element k at byte k),
 *     then in_dim/64 fp16 scales, then in_dim/64 fp16 biases, zero-padded to a
 *     multiple of 16 bytes (moe_qrow_bytes).  w[o][k] = q*scale[k/64] +
 *     bias[k/64]  (affine, group 64).
 *   Expert block (moe_expert_block_bytes(H, I)): 2I gate/up records of H
 *     inputs interleaved gate_0, up_0, gate_1, up_1, ..., then H down records
 *     of I inputs.  Every row, and every run of rows one unit of work needs,
 *     is one contiguous span (one bulk copy / one coalesced warp read).
 * Supported shapes: H a power of two in [256, 4096], I a power of two in
 *   [128, 2048], I_s == I, 1 <= K <= 8, K <= E <= 256, LoRA rank r one of
 *   0 (no adapters), 8, 16, 24, 32 (the adapters move in 16-byte units),
 *   Prerouter E % 8 == 0 and P % 8 == 0, 0 <= T <= MOE_MAX_TOKENS tokens per
 *   call.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Most tokens one call takes: the GEMV kernels walk tokens in passes of 8,
 * one grid row per pass, and a grid has at most 65,535 rows.  A larger T
 * returns MOE_ERR_UNSUPPORTED (workspace queries return 0). */
#define MOE_MAX_TOKENS 524280

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer */
  MOE_ERR_UNSUPPORTED = 2,  /* shape outside the supported set above */
  MOE_ERR_WORKSPACE = 3,    /* workspace smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,         /* a kernel launch failed (cudaGetLastError) */
  MOE_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up */
  MOE_ERR_RANGE = 6         /* an activation outside the fp16 range the kernels compute in (|u| > 65504) */
} moe_status;

/* A quantised matrix stored as out_dim row records (see Formats), 16-byte aligned. */
typedef struct {
  const void* rows;
  int32_t out_dim, in_dim, bits;
} moe_qrows;

/*
 * One routed-expert layer.
 *
 * Routed experts live in one HBM pool: expert e is the expert block at
 * pool + e*expert_stride (expert_stride >= moe_expert_block_bytes(H, I), a
 * multiple of 256).  The shared expert is one more expert block.
 *
 * LoRA (unmerged, 2kiu.com "Recover-LoRA" bullet): the delta on a projection
 * with input x is lora_scale * B (A x), added before the activation; A is
 * [r][in] fp16, B is [out][r] fp16.  Shared expert: index 0 gate, 1 up, 2 down;
 * a NULL A disables that projection's delta.  Routed experts (optional):
 * down projection ex_lora_A [E][r][I], ex_lora_B [E][H][r], or NULL; gate and
 * up projections ex_lora_A_gu [E][2][r][H] (gate's A, then up's A) and
 * ex_lora_B_gu [E][2I][r] in the expert block's interleaved row order (row 2j:
 * gate row j, row 2j+1: up row j), or NULL.  With routed gate/up adapters
 * moe_expert_forward takes its tensor-core path at every T (H and 2I
 * multiples of 128, I of 64; else MOE_ERR_UNSUPPORTED), and moe_stack_decode
 * its per-layer path.
 */
typedef struct {
  int32_t H, E, I, I_s, r;
  moe_qrows router;            /* 8-bit [E][H] */
  const float* router_bias;    /* [E] fp32 added to the logits, or NULL */
  moe_qrows shared_gate;       /* 8-bit [1][H]; g = sigmoid(w . u) */
  const void* shared_block;    /* shared expert, one expert block (I_s == I) */
  const uint16_t* sh_lora_A[3];
  const uint16_t* sh_lora_B[3];
  float lora_scale;
  const void* pool;
  int64_t expert_stride;
  const uint16_t* ex_lora_A;
  const uint16_t* ex_lora_B;
  const uint16_t* ex_lora_A_gu;
  const uint16_t* ex_lora_B_gu;
} moe_layer;

/*
 * Prerouter head (news18a.com Edge0 article, Prerouter paragraph; 2kiu.com
 * "Prerouter" bullet): p = W2 silu(W1 [u ; multi_hot(sel)] + b1) + b2, then the
 * top-K_next of p.  W1 [P][H+E] fp16 (first H columns act on u, last E on the
 * multi-hot of the executed experts), b1 [P], W2 [E_next][P], b2 [E_next] fp16.
 */
typedef struct {
  const uint16_t* W1;
  const uint16_t* b1;
  const uint16_t* W2;
  const uint16_t* b2;
  int32_t H, E, P, E_next;
} moe_prerouter;

/* Human-readable name of a status code (static string, host). */
const char* moe_status_string(moe_status s);

/* Bytes of one row record of in_dim inputs at `bits` (4 or 8); 0 if unsupported (host). */
size_t moe_qrow_bytes(int32_t in_dim, int32_t bits);

/* Bytes of one expert block (host). */
size_t moe_expert_block_bytes(int32_t H, int32_t I);

/*
 * Stack glue between layers (the pages omit attention and norms; this is the
 * plain reading used to stack MoE layers): u[t] = bf16(x[t] / sqrt(mean(x[t]^2)
 * + eps)), computed in fp32.  x [T][H] fp32, u [T][H] bf16.
 */
moe_status moe_rmsnorm_bf16(const float* x, int32_t T, int32_t H, float eps, uint16_t* u, void* stream);

/*
 * Router top-K softmax gating (autoark.ai tier table: K of E routed experts;
 * 2kiu.com config.json paragraph: the router gate is 8-bit).
 *   logits[t][e] = sum_k u[t][k] * W_r[e][k] + router_bias[e]   (fp32)
 *   idx[t][0..K-1] = the K largest logits, descending, equal values -> lower index
 *   w[t][k]  = exp(l_k - l_0) / sum_j exp(l_j - l_0) over the K selected
 * u [T][H] bf16; logits [T][E] fp32 (required output); idx [T][K] int32;
 * w [T][K] fp32.  Two launches.
 * Paths (chosen by shape and alignment only): from 256 tokens on, with E a
 *   multiple of 128 and u 16-byte aligned, the logits come from a tcgen05
 *   GEMM with bf16 operands: per 64-input group the exact products of the
 *   codes minus 128 with u accumulate in fp32 in tensor memory, and each group
 *   is folded in as s*D + (b + 128 s)*sum(u) in fp32 (no weight is rounded;
 *   any finite bf16 u is taken).  Otherwise a dequant-fused GEMV on the CUDA
 *   cores multiplies u rounded to fp16 (see MOE_ERR_RANGE).
 */
moe_status moe_route_topk(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K,
                          float* logits, int32_t* idx, float* w, int32_t* err_word, void* stream);

/*
 * Routed experts + shared expert + combine for T tokens with K experts each
 * (2kiu.com bullets "SSD expert offload" and "Recover-LoRA"; the pool replaces
 * the pages' SSD with HBM):
 *   h_{t,k} = silu(Wg u_t) * (Wu u_t),  y_{t,k} = Wd h_{t,k} (+ routed down LoRA)
 *   for expert e = idx[t][k]; shared expert likewise with its LoRA deltas;
 *   g_t = sigmoid(shared_gate . u_t);
 *   out_t = sum_{k=0}^{K-1} w[t][k] y_{t,k} + g_t y_shared,t   (k order fixed)
 * u [T][H] bf16; idx [T][K] int32 in [0,E) (a value outside is clamped to
 *   0 or E-1, so no read leaves the pool); w [T][K] fp32.
 * out_mode 0: out [T][H] fp32 = result;  1: out [T][H] bf16 = result;
 *          2: out [T][H] fp32 += result (residual stream).
 * perm_out: if not NULL, receives the expert-sorted slot order [T*K] int32
 *   (slot t*K+k; stable, ascending slot id within an expert).
 * workspace: device scratch of at least moe_workspace_size(L, T, K) bytes,
 *   256-byte aligned; its contents on entry do not matter.
 * Paths (chosen by shape only): T*K < 48 slots run dequant-fused GEMVs on the
 *   CUDA cores (fp32 accumulation of exact fp16 x int4-code products); T*K >=
 *   48 slots (with H and 2I multiples of 128) run grouped GEMMs on the tcgen05
 *   tensor cores over per-expert token buckets, where the dequantised weights
 *   and the SwiGLU output are rounded to fp16 and products accumulate in fp32;
 *   there the shared expert's LoRA deltas (scale * B A x per token and output)
 *   are formed in fp32 and rounded to fp16 before they join the accumulator.
 * Bounded waits: every device-side wait of the tensor-core path gives up after
 *   2 s, so a call always completes; a wait that ran out stores MOE_ERR_TIMEOUT
 *   in err_word (see Errors) and leaves the output undefined.
 */
moe_status moe_expert_forward(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K,
                              const int32_t* idx, const float* w, void* out, int32_t out_mode,
                              int32_t* perm_out, void* workspace, size_t ws_bytes, int32_t* err_word,
                              void* stream);

/* Scratch bytes moe_expert_forward needs for (L, T, K) (host); 0 for a NULL
 * layer, T < 0, T > MOE_MAX_TOKENS or K < 1. */
size_t moe_workspace_size(const moe_layer* L, int32_t T, int32_t K);

/*
 * Prerouter prediction (see moe_prerouter).  u [T][H] bf16; sel [T][K] int32
 * = experts executed at this layer, distinct within a row (each entry adds its
 * W1 column once, so distinct entries give the multi-hot product; a value
 * outside [0,E) is clamped to 0 or E-1); pred [T][K_next] int32 (same ordering and
 * tie rule as moe_route_topk); scores [T][E_next] fp32 (required output, the
 * p vector); workspace >= prerouter_workspace_size(head, T) bytes.
 * Paths (chosen by shape and alignment only): from 256 tokens on, with P a
 *   multiple of 128, E of 64 and u 16-byte aligned, the first layer is a
 *   tcgen05 GEMM over [u ; multi_hot(sel)] with W1 split exactly into two bf16
 *   parts (fp32 accumulation, no input rounded); otherwise a GEMV on the CUDA
 *   cores with u rounded to fp16.  The second layer is a CUDA-core GEMV.
 */
moe_status prerouter_predict(const moe_prerouter* head, const uint16_t* u, const int32_t* sel,
                             int32_t T, int32_t K, int32_t K_next, int32_t* pred, float* scores,
                             void* workspace, size_t ws_bytes, int32_t* err_word, void* stream);

/* Scratch bytes prerouter_predict needs for T tokens (host); 0 for a NULL head,
 * T < 0 or T > MOE_MAX_TOKENS. */
size_t prerouter_workspace_size(const moe_prerouter* head, int32_t T);

/*
 * Tiered expert pool (p1 flow and p3 offload: experts sharded on SSD, only the
 * active ones brought into RAM; p2 Prerouter and p3 Prerouter: the head's
 * prediction lets the loads start early).  Here pinned host memory plays the
 * SSD and HBM the RAM: a layer's routed expert blocks live in a host pool,
 * and an HBM cache of n_slots blocks holds the ones in use.  A moe_tier is a
 * host object (least-recently-used replacement; host-to-device copies with
 * cudaMemcpyAsync).  One call of the expert forward over the cache:
 *   moe_tier_acquire   makes the call's experts resident (copies of the missing
 *                      ones on `stream`) and writes the call's expert ids
 *                      remapped to slot ids (idx_slot, device);
 *   moe_expert_forward with a layer view whose pool is the slot array
 *                      (expert_stride = slot_stride, E = n_slots, no routed
 *                      LoRA) and idx = idx_slot, on the same stream;
 *   moe_tier_release   records that the slots' readers so far are enqueued.
 * moe_tier_prefetch starts copies of predicted experts on a second stream (one
 * copy stream per tier); they wait for the last release, never evict the last
 * acquire's experts, and the next acquire waits for them.
 * host_pool: pinned (page-locked or registered) host memory, n_experts blocks
 *   host_stride bytes apart; block_bytes per expert; hbm_slots: device memory
 *   of n_slots blocks, slot_stride bytes apart (>= block_bytes, a multiple of
 *   256, 256-byte aligned); n_experts <= 256.  The caller owns both buffers
 *   and keeps them alive until moe_tier_destroy.  Calls on one tier are
 *   serialised by a lock.  Errors: MOE_ERR_INVALID_ARG for bad pointers or
 *   sizes, MOE_ERR_WORKSPACE when one acquire asks for more distinct experts
 *   than there are slots, MOE_ERR_CUDA when a copy or launch fails; an id in
 *   idx whose expert was not acquired stores MOE_ERR_INVALID_ARG in err_word.
 */
typedef struct moe_tier moe_tier;

typedef struct {
  int64_t acquires;          /* moe_tier_acquire calls */
  int64_t requested;         /* distinct experts asked for, summed over acquires */
  int64_t hits;              /* ... already resident */
  int64_t prefetch_hits;     /* ... of which a prefetch brought in */
  int64_t misses;            /* ... copied by the acquire */
  int64_t prefetched;        /* experts a prefetch copied */
  int64_t bytes_acquired;    /* bytes copied by acquires */
  int64_t bytes_prefetched;  /* bytes copied by prefetches */
} moe_tier_stats;

moe_status moe_tier_create(const void* host_pool, int64_t host_stride, int32_t n_experts, int64_t block_bytes,
                           void* hbm_slots, int64_t slot_stride, int32_t n_slots, moe_tier** out);
void moe_tier_destroy(moe_tier* tier);
/* experts: host array of n_list expert ids (repeats allowed; the call's distinct experts); idx: device
 * [n_idx] expert ids of the call; idx_slot: device [n_idx] output. */
moe_status moe_tier_acquire(moe_tier* tier, const int32_t* experts, int32_t n_list, const int32_t* idx,
                            int32_t n_idx, int32_t* idx_slot, int32_t* err_word, void* stream);
moe_status moe_tier_release(moe_tier* tier, void* stream);
/* experts: host array of n predicted expert ids; at most n_slots distinct ones are copied. */
moe_status moe_tier_prefetch(moe_tier* tier, const int32_t* experts, int32_t n, void* copy_stream);
moe_status moe_tier_get_stats(const moe_tier* tier, moe_tier_stats* out);

/* Options of moe_stack_decode (NULL = all defaults). */
typedef struct {
  int64_t timeout_ns;  /* bound on every device-side wait (single-launch kernel; per-layer grouped GEMMs);
                          <= 0: 1 s for the single launch, 2 s for the GEMMs */
  int32_t path;        /* 0: automatic; 1: per-layer launches; 2: single-launch kernel (MOE_ERR_UNSUPPORTED if
                          the shapes are not eligible); 3: the first-generation single-launch kernel (kept for
                          comparison) */
  int32_t test_drop_layer;  /* test hook for the timeout path, 0 = off; L > 0: on the single-launch path CTA */
  int32_t test_drop_cta;    /*   test_drop_cta never publishes its residual rows of layer L-1, so the other CTAs'
                                 bounded waits run out; on the per-layer path the CTA test_drop_cta of layer L-1's
                                 gate/up grouped GEMM (tensor-core path only) never marks its first operand stage
                                 full, so the MMA's bounded wait runs out.  Either way err_word reports
                                 MOE_ERR_TIMEOUT */
  int64_t* trace;           /* optional device buffer [n_layers][moe_stack_grid()][16] of int64 %globaltimer
                               stamps (ns) per CTA of the single-launch kernel (paths 0 and 2), written by its
                               thread 0: 0 x received, 1 RMSNorm done and layer weights landed, 2 router /
                               shared-gate / LoRA-A rows published, 3 shared (gate, up) dots and Prerouter u part
                               done, 4 logits received, 5 top-K done, 6 routed copies issued, 7 (gate, up) pairs
                               done, 8 hidden values published and previous head's output rows done, 9 hidden
                               vector received, 10 down rows landed, 11 down sub-rows done, 12 x rows published,
                               15 first routed pair landed (if thread 0's warp computes it) */
} moe_stack_opts;

/* Grid size (CTAs) the single-launch stack kernel uses on the current device (host). */
int32_t moe_stack_grid(void);

/*
 * A stack of n_layers routed-expert layers on a residual stream (attention is
 * omitted, as in the pages' statement of the hot path; the norm between
 * layers is the moe_rmsnorm_bf16 glue):
 *   for l: u_l = bf16(rmsnorm(x)); route; x += MoE_l(u_l); pred_l = head_l(u_l, executed_l)
 * With use_predicted_routing (2kiu.com "Prerouter" bullet: the prediction is
 * used directly as the routing), layer l >= 1 executes pred_{l-1} with gating
 * weights = softmax of its own logits at those indices; requires K_next == K.
 * x [T][H] fp32 in/out.  Optional outputs (NULL = not written):
 *   x_trace [n_layers][T][H] fp32 (x entering each layer),
 *   u_trace [n_layers][T][H] bf16, idx_all [n_layers][T][K] executed experts,
 *   true_idx_all [n_layers][T][K] the router's own top-K,
 *   pred_all [n_layers][T][K_next].
 * heads may be NULL (no Prerouter) unless use_predicted_routing.
 * All layers must share H, E, I and r; heads share P and E_next.
 *
 * Paths: for one token (T == 1) without predicted routing, H 1024 or 2048,
 * I 512, shared LoRA on all three projections or none, no routed LoRA and
 * K_next == K, the whole stack runs as ONE cooperative kernel launch (one CTA
 * per SM; layer-internal exchanges through device memory with bounded waits);
 * otherwise as per-layer launches of the kernels behind the per-layer entry
 * points.  err_word (device, optional): set to 0 at the start of the call,
 * then collects the device-side status of every launch of the stack (see
 * Errors): MOE_ERR_TIMEOUT if a bounded wait of the single-launch kernel or of
 * a per-layer grouped GEMM gave up (the outputs are then undefined); read it
 * after synchronising the stream.
 * workspace >= moe_stack_workspace_size(...) bytes, 256-byte aligned; contents
 * on entry do not matter.
 */
moe_status moe_stack_decode(const moe_layer* layers, const moe_prerouter* heads, int32_t n_layers, int32_t T,
                            int32_t K, int32_t K_next, float eps, float* x, float* x_trace, uint16_t* u_trace,
                            int32_t* idx_all, int32_t* true_idx_all, int32_t* pred_all,
                            int32_t use_predicted_routing, int32_t* err_word, const moe_stack_opts* opts,
                            void* workspace, size_t ws_bytes, void* stream);

/* Scratch bytes moe_stack_decode needs (host); 0 for NULL layers,
 * n_layers < 1, T < 0, T > MOE_MAX_TOKENS or K < 1. */
size_t moe_stack_workspace_size(const moe_layer* layers, const moe_prerouter* heads, int32_t n_layers, int32_t T,
                                int32_t K, int32_t K_next);

/*
 * Allocation-free variant of moe_expert_forward.  The pages have no
 * counterpart: this exists for callers that cannot allocate device memory for
 * a workspace -- e.g. a host framework that owns every device allocation and
 * hands a custom operator only its inputs and outputs, or a process whose
 * caching allocator has already reserved nearly all of HBM so that a fresh
 * cudaMalloc would fail.
 *
 * Same computation, arguments and output modes as moe_expert_forward, but the
 * scratch comes from a fixed array of MOE_NOALLOC_SCRATCH_BYTES (4 MiB) in the
 * library's device memory, which every GPU that loads the library reserves
 * until the process exits.  This call itself allocates nothing (no cudaMalloc,
 * no library allocator).
 * Errors: MOE_ERR_WORKSPACE when moe_workspace_size(L, T, K) exceeds
 *   MOE_NOALLOC_SCRATCH_BYTES (nothing is enqueued); otherwise as
 *   moe_expert_forward.
 * Set-up: the first call on a device (with that device current) looks up the
 *   array's device address once and keeps it for the life of the process (a
 *   failed lookup is retried by the next call); make that first call before
 *   any stream capture on that device.  A process that calls cudaDeviceReset
 *   must not use this entry point afterwards: the library's module is then
 *   reloaded, possibly elsewhere, and the kept address is stale.
 * Sharing: all calls in the process share the one array per device and it
 *   keeps the previous call's contents.  Every scratch word the kernels read
 *   is written earlier in the same call, so nothing needs clearing; but calls
 *   that overlap on the GPU (different streams, or different host threads
 *   without ordering) race on the array and must be serialised by the caller.
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

moe_status moe_expert_forward_noalloc(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K,
                                      const int32_t* idx, const float* w, void* out, int32_t out_mode,
                                      int32_t* perm_out, int32_t* err_word, void* stream);

/* MOE_NOALLOC_SCRATCH_BYTES as compiled into the library (host). */
size_t moe_noalloc_scratch_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
