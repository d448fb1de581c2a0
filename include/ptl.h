/*
 * ptl.h -- C ABI of the packed-sequence Transformer layer library (libptl.so).
 *
 * The library runs the forward pass of a pre-norm encoder layer over many
 * users' behaviour sequences packed end to end into one jagged token stream,
 * as described in the "Days-gone/cti2026" README (TransformerEncoder
 * section):
 *
 *     x1  = x  + Linear_out( Attn( LayerNorm1(x) Wqkv^T + b_qkv, user_offsets ) )
 *     out = x1 + FusedMoE( LayerNorm2(x1), Gate(LayerNorm2(x1)) )
 *
 * Attention is block-diagonal causal: token i of a user attends to that
 * user's tokens 0..i only (README, FlashAttention_Varlen operator design).
 * The gate is Linear(512->8) followed by softmax, top-2 and renormalisation
 * (README, SMoE structure); each token's two experts Linear(512->1024) +
 * ReLU + Linear(1024->512) are combined with the renormalised weights
 * (README, fused MoE routing and weighted sum).  The prediction head is a
 * final LayerNorm, Linear(512->1), clamp to [-15, 15] and sigmoid on the
 * tokens whose pred_mask is set (README, Prediction Head section).
 *
 * Layer shape is fixed: d_model 512, 8 heads x 64, QKV 512->1536, gate
 * 512->8, 8 experts 512->1024->512, top-2.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers unless stated otherwise and
 *     row-major.  Activations, weights, biases and LayerNorm parameters must
 *     be 16-byte aligned; topk_idx / topk_w written by ptl_gate 8-byte
 *     aligned; cu_seqlens, perm, expert_off, probs and n_pred 4-byte
 *     aligned (PTL_ERR_ALIGN otherwise).  Weight matrices use the nn.Linear
 *     layout W[out][in].
 *   - Activations and the big matrices (w_qkv, w_o, w1, w2) are stored in
 *     the build dtype `dt`: PTL_BF16 (bfloat16 storage, fp32 accumulation)
 *     or PTL_F32 (fp32 storage and arithmetic).  LayerNorm parameters, the
 *     gate weight and every bias are float32 in both builds.  Bias pointers
 *     may be NULL (treated as zero); LayerNorm gamma/beta may not.
 *   - cu_seqlens (user_offsets) is int32 [num_users + 1] with cu[0] = 0,
 *     non-decreasing, cu[num_users] = total_tokens.  Zero-length users are
 *     allowed anywhere and produce nothing.  These properties are checked on
 *     the device; a violation sets the workspace error word to
 *     PTL_ERR_BAD_OFFSETS, later kernels of the call skip their work, the
 *     outputs are undefined, and ptl_last_device_error() reports it.
 *   - The caller owns every buffer.  The library allocates nothing inside
 *     the forward calls, never synchronises `stream` and keeps no state
 *     between calls, so a sequence of calls can be captured into a CUDA
 *     graph (TMA descriptors are built on the host at call time and passed
 *     by value, so a captured graph keeps the buffers it was captured on).
 *     `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   - workspace: a device buffer of at least ptl_workspace_size(T, U, dt)
 *     bytes, 256-byte aligned, used only by the calls that receive it.  Two
 *     calls that run concurrently must not share a workspace.  Its contents
 *     need no initialisation for the calls (each clears the error word before
 *     its first launch); ptl_last_device_error on a workspace that no call has
 *     used reads whatever its first word holds, so zero a new one first.
 *   - Host-checkable problems (NULL pointers, misalignment, sizes, a too
 *     small workspace, an unknown dtype) return a status immediately and
 *     launch nothing.  total_tokens == 0 returns PTL_OK with no launches.
 *     No entry point traps, prints or throws across the ABI.
 */
#ifndef PTL_H
#define PTL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PTL_D_MODEL 512
#define PTL_N_HEADS 8
#define PTL_D_HEAD 64
#define PTL_D_FF 1024
#define PTL_N_EXPERTS 8
#define PTL_TOP_K 2

typedef enum {
  PTL_OK = 0,
  PTL_ERR_NULL = 1,        /* a required pointer is NULL */
  PTL_ERR_ALIGN = 2,       /* a pointer is not 16-byte aligned (workspace: 256) */
  PTL_ERR_SHAPE = 3,       /* num_users < 1, total_tokens < 0 or >= 2^31, num_layers < 1 */
  PTL_ERR_BAD_OFFSETS = 4, /* cu_seqlens not 0-based, not monotone, or not ending at T */
  PTL_ERR_WORKSPACE = 5,   /* workspace smaller than ptl_workspace_size() */
  PTL_ERR_DTYPE = 6,       /* unknown ptl_dtype */
  PTL_ERR_CUDA = 7,        /* a CUDA runtime call or launch failed */
  PTL_ERR_TIMEOUT = 8,     /* a bounded device-side wait ran out (kernel returned early) */
  PTL_ERR_UNSUPPORTED = 9, /* no sm_100 device, or a feature not built */
  PTL_ERR_BAD_MASK = 10,   /* attention mask out of range (ptl_attention_masked) */
  PTL_ERR_BAD_IDS = 11     /* embedding id outside its table or bad bag offsets (ptl_rep_encoder) */
} ptl_status;

typedef enum { PTL_F32 = 0, PTL_BF16 = 1 } ptl_dtype;

/* One layer's parameters (device pointers). */
typedef struct {
  const void* ln1_g;  /* [512] f32 */
  const void* ln1_b;  /* [512] f32 */
  const void* w_qkv;  /* [1536][512] dt; rows 0-511 Q, 512-1023 K, 1024-1535 V; head h = rows 64h..64h+63 of each */
  const void* b_qkv;  /* [1536] f32 or NULL */
  const void* w_o;    /* [512][512] dt */
  const void* b_o;    /* [512] f32 or NULL */
  const void* ln2_g;  /* [512] f32 */
  const void* ln2_b;  /* [512] f32 */
  const void* w_gate; /* [8][512] f32 */
  const void* b_gate; /* [8] f32 or NULL */
  const void* w1;     /* [8][1024][512] dt */
  const void* b1;     /* [8][1024] f32 or NULL */
  const void* w2;     /* [8][512][1024] dt */
  const void* b2;     /* [8][512] f32 or NULL */
} ptl_layer_weights;

/* Prediction head parameters (device pointers, all f32). */
typedef struct {
  const void* lnf_g; /* [512] */
  const void* lnf_b; /* [512] */
  const void* w;     /* [512] */
  const void* b;     /* [1] or NULL */
} ptl_head_weights;

/* Optional debug outputs of ptl_layer_forward (device pointers; any may be NULL). */
typedef struct {
  int32_t* topk_idx;   /* [T][2] chosen experts, slot 0 = larger probability */
  float* topk_w;       /* [T][2] renormalised weights */
  int32_t* perm;       /* [2T] routes r = 2t+k sorted by expert, ascending r within an expert */
  int32_t* expert_off; /* [9] exclusive prefix of routes per expert */
} ptl_debug_out;

/* Bytes of workspace needed for calls with up to max_tokens tokens and
 * max_users users in build dtype dt (0 for invalid arguments). */
size_t ptl_workspace_size(int64_t max_tokens, int32_t max_users, ptl_dtype dt);

/* One encoder layer: out[T][512] = layer(x[T][512]).  x and out may not
 * alias.  dbg may be NULL. */
ptl_status ptl_layer_forward(const void* x, void* out, const int32_t* cu_seqlens,
                             int32_t num_users, int64_t total_tokens, ptl_dtype dt,
                             const ptl_layer_weights* w, void* workspace, size_t ws_bytes,
                             const ptl_debug_out* dbg, void* stream);

/* num_layers layers in sequence (layers: HOST array of num_layers structs
 * holding device pointers), then, when head != NULL, the prediction head:
 * probs[0 .. n_pred-1] = sigmoid(clamp(LN_f(h) w + b)) for the tokens with
 * pred_mask[t] != 0 in ascending t; *n_pred (device int32) receives the
 * count.  out[T][512] always receives the final hidden state.  With head ==
 * NULL, pred_mask/probs/n_pred are ignored.  x and out may not alias. */
ptl_status ptl_stack_forward(const void* x, void* out, const int32_t* cu_seqlens,
                             int32_t num_users, int64_t total_tokens, int32_t num_layers,
                             ptl_dtype dt, const ptl_layer_weights* layers,
                             const ptl_head_weights* head, const uint8_t* pred_mask,
                             float* probs, int32_t* n_pred, void* workspace, size_t ws_bytes,
                             void* stream);

/* ---- The layer's steps, one entry point each (the cti2026 README's operator
 * interface: Linear_qkv, FlashAttention_Varlen(qkv, user_offsets),
 * Linear_out + residual, Gate(x) -> (topk_idx, topk_weight),
 * FusedMoE(x, topk_idx, topk_weight) + residual, Prediction Head). ---- */

/* qkv[T][1536] = LayerNorm1(x) Wqkv^T + b_qkv (uses ln1_g, ln1_b, w_qkv, b_qkv of w). */
ptl_status ptl_qkv_projection(const void* x, void* qkv, int64_t total_tokens, ptl_dtype dt,
                              const ptl_layer_weights* w, void* workspace, size_t ws_bytes,
                              void* stream);

/* attn[T][512] = block-diagonal causal softmax(Q K^T / 8) V per user and head,
 * Q/K/V read from qkv[T][1536] as [Q|K|V]. */
ptl_status ptl_attention(const void* qkv, void* attn, const int32_t* cu_seqlens,
                         int32_t num_users, int64_t total_tokens, ptl_dtype dt,
                         void* workspace, size_t ws_bytes, void* stream);

/* x1[T][512] = x + attn Wo^T + b_o.  x1 is float32 in both builds: the
 * residual stream inside a layer is kept in fp32 so that the layer output is
 * rounded to the build dtype once. */
ptl_status ptl_out_projection(const void* attn, const void* x, void* x1, int64_t total_tokens,
                              ptl_dtype dt, const ptl_layer_weights* w, void* workspace,
                              size_t ws_bytes, void* stream);

/* x1: float32 [T][512] (see ptl_out_projection).
 * xn2[T][512] = LayerNorm2(x1) (dt); p = softmax(xn2 Wg^T + bg) in fp32;
 * topk_idx[T][2] (int32) = the two largest p (ties to the lower expert
 * index, slot 0 the larger), topk_w[T][2] (f32) = p / (p0 + p1). */
ptl_status ptl_gate(const void* x1, void* xn2, int32_t* topk_idx, float* topk_w,
                    int64_t total_tokens, ptl_dtype dt, const ptl_layer_weights* w,
                    void* workspace, size_t ws_bytes, void* stream);

/* Counting sort of the 2T routes r = 2t+k by topk_idx: expert_off[9] is the
 * exclusive prefix of the per-expert counts and perm[2T] lists the routes of
 * expert 0, then expert 1, ..., each in ascending r.  Either output may be
 * NULL.  topk_idx values must be in [0, 8). */
ptl_status ptl_route_build(const int32_t* topk_idx, int64_t total_tokens, int32_t* perm,
                           int32_t* expert_off, void* workspace, size_t ws_bytes, void* stream);

/* residual: float32 [T][512] (x1 of the layer); out: [T][512] in dt.
 * out[t] = residual[t] + topk_w[t][0] y(t, topk_idx[t][0]) + topk_w[t][1] y(t, topk_idx[t][1]),
 * y(t, e) = ReLU(xn2[t] W1[e]^T + b1[e]) W2[e]^T + b2[e]  (uses w1, b1, w2, b2 of w).
 * The k = 0 term is added first, in fp32, and rounded once. */
ptl_status ptl_moe(const void* xn2, const int32_t* topk_idx, const float* topk_w,
                   const void* residual, void* out, int64_t total_tokens, ptl_dtype dt,
                   const ptl_layer_weights* w, void* workspace, size_t ws_bytes, void* stream);

/* Prediction head on h[T][512] (dt), see ptl_stack_forward. */
ptl_status ptl_head(const void* h, const ptl_head_weights* head, const uint8_t* pred_mask,
                    float* probs, int32_t* n_pred, int64_t total_tokens, ptl_dtype dt,
                    void* workspace, size_t ws_bytes, void* stream);

/* ---- HSTU-style attention masks over the same jagged layout. ----
 * The cry-daniel/recsys README (HSTU attention mask logic) lays a user's
 * sequence out as [contextual tokens][historical tokens][candidate tokens]:
 * contextual tokens (user profile) attend to one another in both
 * directions, history is causal, candidates are grouped by
 * target_group_size; its attention function also offers no mask and a local
 * (sliding-window) mask.  For the user with L tokens, C = num_contexts[u]
 * and N = num_targets[u] (candidates from Hs = L - N), key j is visible to
 * query i when
 *   (causal ? j <= i : 1)  or  (i < C and j < C),
 *   and, if j >= Hs: i >= Hs and (i - Hs) / G == (j - Hs) / G,
 *   and, if window > 0: |i - j| < window.
 * Every query sees itself.  ptl_attention_masked computes softmax(Q K^T / 8) V
 * per user and head over the visible keys, reading Q/K/V from qkv[T][1536]
 * like ptl_attention; with causal = 1 and no contexts, candidates or window
 * it equals ptl_attention.  num_contexts / num_targets: device int32 [U],
 * NULL = all zero.  Host checks: target_group_size >= 1 and causal 0 or 1
 * (else PTL_ERR_BAD_MASK), plus the usual ones; on the device, a user with
 * C < 0, N < 0 or C + N > L sets PTL_ERR_BAD_MASK in the workspace error
 * word (the attention then computes nothing). */
typedef struct {
  int32_t causal;             /* 1: causal base rule; 0: every key of the user (no mask) */
  const int32_t* num_contexts; /* device [U] or NULL */
  const int32_t* num_targets;  /* device [U] or NULL */
  int32_t target_group_size;  /* candidates per group, >= 1 */
  int32_t window;             /* > 0: sliding window |i - j| < window; <= 0: none */
} ptl_attn_mask;
ptl_status ptl_attention_masked(const void* qkv, void* attn, const int32_t* cu_seqlens,
                                int32_t num_users, int64_t total_tokens, ptl_dtype dt,
                                const ptl_attn_mask* mask, void* workspace, size_t ws_bytes,
                                void* stream);

/* ---- Per-kernel tracing (for profiling; off by default). ----
 * While a trace is installed on the calling host thread, every entry point
 * records events[count] on its stream just before each kernel (or memset)
 * it enqueues, stores that launch's kind in kinds[count] and increments
 * count; after its last launch it records one more event with kind
 * PTL_KERNEL_END.  The time of launch i is the elapsed time between
 * events[i] and events[i + 1].  events are cudaEvent_t handles created by
 * the caller (with timing enabled); kinds is a host array.  Recording stops
 * silently when count reaches capacity.  The trace is owned by the caller
 * and must outlive the calls it observes; pass NULL to remove it. */
typedef enum {
  PTL_KERNEL_CLEAR = 0,        /* error-word / counter memsets */
  PTL_KERNEL_WORKLIST = 1,     /* cu_seqlens validation + attention work list */
  PTL_KERNEL_LAYERNORM = 2,    /* LayerNorm1 */
  PTL_KERNEL_GEMM_QKV = 3,     /* QKV projection */
  PTL_KERNEL_ATTENTION = 4,    /* jagged causal attention */
  PTL_KERNEL_GEMM_OUT = 5,     /* output projection + residual */
  PTL_KERNEL_GATE = 6,         /* LayerNorm2 + gate + top-2 */
  PTL_KERNEL_ROUTE = 7,        /* route counting sort (and per-chunk counts) */
  PTL_KERNEL_GEMM_EXPERT1 = 8, /* expert GEMM1 + ReLU (gathered rows) */
  PTL_KERNEL_GEMM_EXPERT2 = 9, /* expert GEMM2 (per-route outputs) */
  PTL_KERNEL_HEAD = 10,        /* prediction head + compaction */
  PTL_KERNEL_COPY = 11,        /* debug-output copies */
  PTL_KERNEL_COMBINE = 12,     /* weighted top-2 combine + residual */
  PTL_KERNEL_END = 99
} ptl_kernel_kind;

typedef struct {
  void** events;    /* cudaEvent_t[capacity] */
  int32_t* kinds;   /* host [capacity] */
  int32_t capacity;
  int32_t count;
} ptl_trace;

/* Installs (or, with NULL, removes) the calling thread's trace. */
void ptl_set_trace(ptl_trace* trace);

/* ---- Attention without any device allocation. ----
 * Some callers cannot allocate device memory: host programs that own all of
 * device memory through their own pool or budget and hand a library no
 * allocator, and latency-critical loops that cannot afford cudaMalloc, which
 * may synchronise the whole device.  ptl_attention_noalloc computes what
 * ptl_attention computes (same arguments, no workspace): its only scratch,
 * the device error word and the attention work list (the (user, query
 * block) pairs and each attention CTA's unit lists), lives in one fixed
 * array of PTL_NOALLOC_SCRATCH_BYTES bytes in the library's device memory,
 * which every GPU that loads the library holds until the process exits.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Limits: total_tokens <= PTL_NOALLOC_MAX_TOKENS and num_users <=
 *     PTL_NOALLOC_MAX_USERS; larger requests return PTL_ERR_SHAPE and launch
 *     nothing.
 *   - The first call on each device is its set-up: it looks up the array's
 *     device address (cudaGetSymbolAddress, with that device current) and
 *     caches it.  With lazy module loading (the CUDA 12 default) that lookup
 *     is also what loads the library's kernels onto the device and backs the
 *     array, which may reserve device memory and synchronise; every later
 *     call reuses the cached address and reserves nothing.  Make the first
 *     call before any stream capture.  The cached address belongs to the
 *     device's current context: after cudaDeviceReset in the same process it
 *     is stale, so do not call this entry point on a device that was reset.
 *   - Every call on a device uses the same array, which keeps the previous
 *     call's contents (each call clears what must start at zero).  Calls
 *     that can overlap on the GPU -- on different streams with no ordering
 *     between them -- race on the array; do not issue them.
 *   - device_status (nullable, device int32, 4-byte aligned) receives the
 *     call's device-side status: PTL_OK, or PTL_ERR_BAD_OFFSETS for a
 *     cu_seqlens that is not 0-based, non-decreasing and ending at T.
 * The pages describe no such entry point; it has no counterpart there. */
#define PTL_NOALLOC_MAX_TOKENS 65536
#define PTL_NOALLOC_MAX_USERS 4096
#define PTL_NOALLOC_SCRATCH_BYTES 655360
ptl_status ptl_attention_noalloc(const void* qkv, void* attn, const int32_t* cu_seqlens,
                                 int32_t num_users, int64_t total_tokens, ptl_dtype dt,
                                 int32_t* device_status, void* stream);

/* ---- The stack as one CUDA graph per token bucket. ----
 * Serving issues the stack batch after batch with a different packing each
 * time.  Issued kernel by kernel that loop is bound by launch overhead
 * (README, CUDA Graph section: about 211 launches per batch); the remedy
 * there is to pad every batch to a bucket of the token count (512-token
 * steps), capture one graph per bucket lazily or ahead of time over static
 * buffers, pad a short batch's user offsets on the GPU with zero-length
 * users, and never synchronise the host.  A runner does that:
 *   - ptl_runner_create allocates, once, a workspace and static input /
 *     output buffers for batches of up to max_tokens tokens and max_users
 *     users (device memory of the current device; the only allocation).
 *     `layers` (num_layers entries) and `head` (nullable) are copied by value;
 *     the device weights they point to must outlive the runner.  stride is
 *     the bucket granule in tokens, a multiple of 128 (0 = PTL_RUNNER_STRIDE).
 *   - ptl_runner_forward computes what ptl_stack_forward computes for the
 *     batch (x [T][512] of the runner's dtype, cu_seqlens [U+1] int32,
 *     pred_mask [T] uint8) with T rounded up to the bucket Tb: it copies the
 *     inputs into the
 *     static buffers (x, cu_seqlens and pred_mask may be host or device
 *     pointers; host memory should be pinned for the copies to be
 *     asynchronous), zero-fills the padding tokens, appends padding users of
 *     at most 128 tokens over T .. Tb and zero-length users up to the
 *     runner's fixed user count (ptl_runner_bucket), launches the bucket's
 *     graph and copies out[T][512] (nullable when there is a head),
 *     probs[0 .. T-1] (entries past *n_pred undefined) and *n_pred (nullable)
 *     to host or device memory.  Real rows equal those of a direct
 *     ptl_stack_forward call on the unpadded batch bit for bit (users are
 *     independent, every other step is per token).  The first batch of a
 *     bucket captures and instantiates its graph (host work, no device
 *     synchronisation; ptl_runner_capture does it ahead of time).  All
 *     work is enqueued on `stream`; a runner's calls must be ordered on one
 *     stream (its buffers are reused by the next batch).  T == 0 returns
 *     PTL_OK without work; T > max_tokens, U > max_users or a call from
 *     another device return PTL_ERR_SHAPE.  Malformed offsets (including
 *     cu_seqlens[U] != T) are reported by ptl_runner_last_device_error as
 *     PTL_ERR_BAD_OFFSETS.
 *   - ptl_runner_destroy frees everything (cudaFree waits for the device).
 * ptl_runner_bucket is host arithmetic only: the bucket of a token count and
 * the runner's padded user count. */
#define PTL_RUNNER_STRIDE 512
typedef struct ptl_stack_runner ptl_stack_runner;
ptl_status ptl_runner_bucket(int64_t total_tokens, int32_t max_users, int32_t stride,
                             int64_t* bucket, int32_t* padded_users);
ptl_status ptl_runner_create(int64_t max_tokens, int32_t max_users, int32_t num_layers, ptl_dtype dt,
                             const ptl_layer_weights* layers, const ptl_head_weights* head,
                             int32_t stride, ptl_stack_runner** runner);
ptl_status ptl_runner_capture(ptl_stack_runner* runner, int64_t total_tokens);
ptl_status ptl_runner_forward(ptl_stack_runner* runner, const void* x, void* out,
                              const int32_t* cu_seqlens, int32_t num_users, int64_t total_tokens,
                              const uint8_t* pred_mask, float* probs, int32_t* n_pred, void* stream);
/* Synchronises `stream`, returns and clears the runner's device error word. */
ptl_status ptl_runner_last_device_error(ptl_stack_runner* runner, void* stream);
/* Number of buckets whose graph has been captured (-1 for NULL). */
int32_t ptl_runner_graphs(const ptl_stack_runner* runner);
void ptl_runner_destroy(ptl_stack_runner* runner);

/* ---- RepEncoder front end. ----
 * The encoder's input rows come from a RepEncoder (cti2026 README,
 * RepEncoder section): for every token, 28 slots each look up a bag of
 * feature ids in their own embedding table and sum the rows (sum pooling;
 * one launch for all slots, the tables passed as 28 pointers, 64-bit row
 * offsets), the [28][512] sums are flattened to 14336 values, normalised by
 * one LayerNorm over those 14336 values (eps 1e-5, biased variance), and
 * Linear(14336 -> 512) gives the token's row:
 *   out[t] = LN(concat_s sum_{i in bag(t, s)} tables[s][ids[i]]) W^T + b.
 * Bag (t, s) holds ids[bag_offsets[t*28 + s] .. bag_offsets[t*28 + s + 1]);
 * an empty bag gives zeros.  ids: device int64 [num_ids]; bag_offsets:
 * device int64 [T*28 + 1], non-decreasing within 0 .. num_ids; out: device
 * [T][512] of dt.  Tables and W in dt, LayerNorm parameters and b in fp32.
 * Device checks: an id outside 0 .. vocab[s]-1, or a bag range outside
 * 0 .. num_ids or decreasing, sets PTL_ERR_BAD_IDS in the workspace error
 * word (read with ptl_last_device_error); the output is then undefined.
 * workspace: ptl_rep_encoder_workspace_size(T, dt) bytes, 256-byte aligned
 * (the error word and the normalised rows).  Asynchronous on `stream`. */
#define PTL_REP_SLOTS 28
typedef struct {
  const void* tables[PTL_REP_SLOTS]; /* device [vocab[s]][512] dt (NULL allowed when vocab[s] == 0) */
  int64_t vocab[PTL_REP_SLOTS];      /* rows of each table */
  const float* ln_g;                 /* [14336] f32 */
  const float* ln_b;                 /* [14336] f32 */
  const void* w;                     /* [512][14336] dt */
  const float* b;                    /* [512] f32 or NULL */
} ptl_rep_encoder_weights;
size_t ptl_rep_encoder_workspace_size(int64_t max_tokens, ptl_dtype dt);
ptl_status ptl_rep_encoder(const int64_t* ids, int64_t num_ids, const int64_t* bag_offsets,
                           int64_t total_tokens, ptl_dtype dt, const ptl_rep_encoder_weights* w,
                           void* out, void* workspace, size_t ws_bytes, void* stream);

/* ---- FP8 (e4m3) linear layers. ----
 * Low-precision GEMMs for the layer's projections (cry-daniel/recsys README:
 * FP8 in its feature list; the CTI-Inference-Opt optimisation plan's INT8
 * section as the motivation).  The pages fix no recipe; the reading taken is
 * e4m3 codes (4 exponent bits, bias 7, 3 mantissa bits, largest finite 448)
 * with one float32 scale per row of each operand: rows of the activations
 * (tokens) and rows of the weight (output channels).
 * ptl_quantize_rows_e4m3: scales[r] = max_c |x[r][c]| / 448 (1 for an
 *   all-zero row) and codes[r][c] = e4m3(x[r][c] / scales[r]), both the scale
 *   and the quotient IEEE float32 operations (correctly rounded), the code
 *   rounded to the nearest e4m3 value, ties to even, saturating at +-448.
 *   x: device [rows][cols] in dt; codes: device uint8 [rows][cols]; scales:
 *   device float [rows].  cols a multiple of 16 (>= 16), x and codes 16-byte
 *   aligned, scales 4-byte aligned.  Asynchronous on `stream`.
 * ptl_linear_fp8: out[m][n] = bf16((sum_k xq[m][k] wq[n][k]) * sx[m] * sw[n]
 *   + b[n]): the code products summed in float32 on the tensor cores
 *   (tcgen05 kind::f8f6f4, 256 x 256 tiles on CTA pairs), then scaled.
 *   xq [M][K] with sx [M] and wq [N][K] with sw [N] as ptl_quantize_rows_e4m3
 *   writes them; bias (nullable) float [N]; out device bf16 [M][N].  K a
 *   multiple of 128, N a multiple of 256, M < 2^31; codes and out 16-byte
 *   aligned.  workspace: >= 256 bytes, 256-byte aligned (its error word, read
 *   by ptl_last_device_error: PTL_ERR_TIMEOUT if a bounded wait ran out).
 *   PTL_ERR_SHAPE for other sizes; M == 0 returns PTL_OK with no launch. */
ptl_status ptl_quantize_rows_e4m3(const void* x, ptl_dtype dt, int64_t rows, int32_t cols, uint8_t* codes,
                                  float* scales, void* stream);
ptl_status ptl_linear_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                          const float* bias, void* out, int64_t rows, int32_t in_features,
                          int32_t out_features, void* workspace, size_t ws_bytes, void* stream);

/* ---- One batch split across GPUs. ----
 * Users are independent (a token attends only to its own user's tokens, and
 * every other step works token by token: cti2026 README, packed batch with
 * user_offsets and the FlashAttention_Varlen design), so one batch splits
 * into contiguous user ranges, one per GPU; each GPU runs the single-GPU
 * entry points on its range with rebased offsets cu_seqlens[b .. e] -
 * cu_seqlens[b] and rows cu_seqlens[b] .. cu_seqlens[e] - 1, and the parts'
 * outputs (rows, or compacted head probabilities, both in ascending token
 * order) concatenated in part order equal the whole batch's.
 * ptl_partition_users chooses the ranges: part r gets users user_begin[r] ..
 * user_begin[r + 1] - 1.  A user of L tokens costs 6,299,648 L (one layer's
 * GEMM FLOPs per token) + 1024 L (L + 1) (its attention FLOPs); the split
 * minimises the largest part's cost over all contiguous splits (the smallest
 * feasible bound, found by bisection over a greedy fill), then fills parts
 * left to right up to that bound, so trailing parts may be empty when there
 * are more parts than users.  Host arithmetic only (no GPU, no allocation).
 *   cu_seqlens: HOST int32 [num_users + 1], 0-based and non-decreasing
 *               (PTL_ERR_BAD_OFFSETS otherwise);
 *   user_begin: HOST int32 [num_parts + 1], written: user_begin[0] = 0,
 *               user_begin[num_parts] = num_users, non-decreasing.
 * PTL_ERR_NULL for a NULL pointer, PTL_ERR_SHAPE for num_users < 1 or
 * num_parts < 1. */
ptl_status ptl_partition_users(const int32_t* cu_seqlens, int32_t num_users, int32_t num_parts,
                               int32_t* user_begin);

/* ---- Failure detection self-test. ----
 * Every wait inside the library's kernels (on an mbarrier phase, or on a
 * counter that another CTA of the same launch raises) is bounded: after a
 * limit without progress the waiting thread records PTL_ERR_TIMEOUT in the
 * workspace error word and its kernel unwinds, leaving the context usable.
 * ptl_wait_selftest launches one 32-thread kernel that runs those same waits
 * on something that never happens -- which = 0: an mbarrier phase that no
 * thread completes; which = 1: a flag in the workspace's error block that is
 * zeroed first and that nothing raises -- so that the give-up path can be run
 * on purpose.  limit_ns (1e3 .. 1e9) replaces the library's one-second limit.
 * Asynchronous on `stream`; afterwards ptl_last_device_error() reports
 * PTL_ERR_TIMEOUT.  Returns PTL_ERR_SHAPE for another `which` or a limit
 * outside the range, and the usual NULL / alignment / size statuses for the
 * workspace (at least 256 bytes). */
ptl_status ptl_wait_selftest(void* workspace, size_t ws_bytes, int32_t which, int64_t limit_ns,
                             void* stream);

/* Synchronises `stream`, returns the status recorded in the workspace error
 * word by earlier calls on that workspace (PTL_OK if none) and clears it. */
ptl_status ptl_last_device_error(void* workspace, size_t ws_bytes, void* stream);

/* Static text for a status code. */
const char* ptl_status_string(ptl_status s);

/* Library ABI version (major * 100 + minor); PTL_VERSION is the value this
 * header describes.  Minor 1 added the graph runner, the masked attention, the
 * RepEncoder front end, the wait self-test and the PTL_ERR_BAD_MASK /
 * PTL_ERR_BAD_IDS codes; minor 2 the user partitioner and the FP8 linear layers. */
#define PTL_VERSION 102
int32_t ptl_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PTL_H */
