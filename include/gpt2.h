/*
 * gpt2.h — C ABI of the B200 GPT-2 training-step library (libgpt2_b200.so).
 *
 * One training step of a decoder-only GPT-2: token + position embedding,
 * pre-LN transformer blocks (LayerNorm, QKV projection with bias, causal
 * multi-head attention, output projection, 4x feed-forward with tanh GELU,
 * residual adds), a final LayerNorm, an LM head tied to the token embedding,
 * mean next-token cross-entropy, the backward pass, global grad-norm clipping
 * and AdamW with decoupled weight decay and bias correction.  Every step runs
 * in hand-written sm_100a CUDA kernels; there is no CPU path.
 *
 * Sources the operations follow (cited by page and section):
 *   [LECTURE] "Andrej Karpathy: reproducing GPT-2 from scratch" (lecture
 *             summary, youtublog.net): architecture, tied head, padded
 *             vocabulary, mixed precision, decay groups, clipping.
 *   [CH28]    "Chapter 28: data, evaluation and recovery" (book.ozine.me),
 *             §28.3 batches of B*T+1 tokens, §28.4 validation loss.
 *   [CS336]   "CS336 from scratch — pretraining" (fengye404.top), §1
 *             cross-entropy, §2 AdamW and gradient clipping.
 *   [ZERO]    "GPT training" (Zero framework docs, ismantic.github.io):
 *             autoregressive objective, model sections, training loop.
 *
 * Conventions for every entry point
 *   - Return value: GPT2_OK (0) or one of the GPT2_ERR_* codes below.  No C++
 *     exception crosses the ABI.  gpt2_last_error() gives a message.
 *   - "device" pointers are CUDA device (or managed) addresses on the device
 *     that was current at gpt2_create; "host" pointers are CPU addresses
 *     (pinned or pageable).  The caller keeps ownership of every pointer it
 *     passes; the library never frees them.
 *   - Work is enqueued on the caller's stream (gpt2_config.stream) and is
 *     asynchronous, except where a host scalar is returned (loss, grad norm)
 *     or a host buffer is read/written: those calls synchronise that stream.
 *   - Matrices are row-major.  Linear weights are [out, in] and a linear
 *     layer computes y = x W^T + b.
 *   - Not thread-safe: one handle is used by one host thread at a time.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define GPT2_OK 0
#define GPT2_ERR_ARG 1          /* bad config/argument, size above capacity */
#define GPT2_ERR_TOKEN 2        /* a token or target id outside [0, vocab_size) */
#define GPT2_ERR_NONFINITE 3    /* non-finite loss or gradient norm: update skipped */
#define GPT2_ERR_CUDA 4         /* a CUDA runtime call failed */
#define GPT2_ERR_OOM 5          /* device allocation failed */
#define GPT2_ERR_TIMEOUT 6      /* a bounded device wait gave up (kernel reported it) */
#define GPT2_ERR_STATE 7        /* calls out of order (e.g. backward without forward) */

/* tensor selectors for gpt2_get_tensor / gpt2_set_tensor */
#define GPT2_PARAM 0            /* fp32 master weights */
#define GPT2_GRAD 1             /* fp32 gradients */
#define GPT2_ADAM_M 2           /* fp32 first moment */
#define GPT2_ADAM_V 3           /* fp32 second moment */

/* element types of op-level buffers */
#define GPT2_F32 0
#define GPT2_BF16 1

typedef struct gpt2_handle gpt2_handle;

/* Device allocator hooks: when alloc is non-NULL every device buffer the
 * handle owns comes from alloc(bytes, ctx) and goes back through
 * free(ptr, ctx) (e.g. PyTorch's caching allocator); otherwise cudaMalloc. */
typedef void* (*gpt2_alloc_fn)(size_t bytes, void* ctx);
typedef void (*gpt2_free_fn)(void* ptr, void* ctx);

typedef struct {
  int n_layer;       /* L  (12 for GPT-2 124M) */
  int n_embd;        /* C  (768); must be a multiple of n_head and of 8 */
  int n_head;        /* H  (12); head size D = C/H must be 16, 32, 64 or 128 */
  int vocab_size;    /* V  (50257): ids a token or target may take */
  int padded_vocab;  /* Vp >= V (50304): rows of the tied matrix; the extra
                        rows are real columns of the output softmax [LECTURE:
                        vocabulary padding] */
  int max_T;         /* rows of the position-embedding matrix (1024) */
  int bf16;          /* 1: bf16 GEMM operands and activations with fp32
                        accumulation, statistics, loss, gradients, master
                        weights and Adam state [LECTURE: mixed precision];
                        0: fp32 everywhere (parity mode, SIMT kernels) */
  float ln_eps;      /* LayerNorm epsilon (1e-5) */
  int max_B;         /* activation capacity: every call needs B <= max_B ... */
  int max_Tseq;      /* ... and T <= max_Tseq <= max_T */
  int resid_init_scale; /* reserved, must be 0 (initial values come from the caller) */
  void* stream;      /* cudaStream_t owned by the caller; NULL = default stream */
  gpt2_alloc_fn alloc; /* optional device allocator, see above */
  gpt2_free_fn free;
  void* alloc_ctx;
} gpt2_config;

/* ---------------------------------------------------------------- handle */

/* Creates a model: validates cfg, allocates the fp32 parameter, gradient and
 * AdamW arenas (zeroed; parameters must then be set with gpt2_set_tensor),
 * the bf16 weight mirrors and the activation/workspace memory for
 * max_B x max_Tseq tokens.  *out receives the handle (NULL on failure; the
 * message is then in gpt2_last_error(NULL)).  Adam's step counter starts at 0. */
int gpt2_create(const gpt2_config* cfg, gpt2_handle** out);

/* Synchronises the stream and frees everything the handle owns. */
int gpt2_destroy(gpt2_handle* h);

/* Last error message of h (or of the last failed gpt2_create when h is NULL).
 * The string lives until the next call on h. */
const char* gpt2_last_error(const gpt2_handle* h);

/* Parameter tensors, in the order [LECTURE: module naming]:
 *   wte [Vp,C], wpe [max_T,C], then for l in 0..L-1: h.l.ln1.w [C], h.l.ln1.b [C],
 *   h.l.attn.qkv.w [3C,C], h.l.attn.qkv.b [3C], h.l.attn.proj.w [C,C],
 *   h.l.attn.proj.b [C], h.l.ln2.w [C], h.l.ln2.b [C], h.l.mlp.fc.w [4C,C],
 *   h.l.mlp.fc.b [4C], h.l.mlp.proj.w [C,4C], h.l.mlp.proj.b [C]; then
 *   lnf.w [C], lnf.b [C].
 * The QKV rows stack q, k, v; head h owns channels [hD, (h+1)D).
 * decay = 1 for 2-D tensors (weight decay applies), 0 for vectors [LECTURE:
 * weight decay on matrices, not on biases or other 1-D parameters].
 * *name stays valid for the handle's lifetime; shape[1] = 1 for vectors. */
int gpt2_num_tensors(const gpt2_handle* h, int* n);
int gpt2_tensor_info(const gpt2_handle* h, int i, const char** name, int* ndim,
                     int64_t shape[2], int* decay);
int gpt2_param_count(const gpt2_handle* h, int64_t* n);

/* Copies tensor i of the selected arena (GPT2_PARAM/GRAD/ADAM_M/ADAM_V) from /
 * to a dense row-major fp32 buffer of the tensor's shape, on the host
 * (on_device = 0; the call synchronises) or on the device (on_device = 1).
 * Setting parameters refreshes the bf16 mirrors before the next forward.
 * Reading GPT2_GRAD after gpt2_zero_grad returns zeros. */
int gpt2_set_tensor(gpt2_handle* h, int i, int which, const float* src, int on_device);
int gpt2_get_tensor(gpt2_handle* h, int i, int which, float* dst, int on_device);

/* AdamW step counter t (number of updates done; the next update uses t+1). */
int gpt2_get_step(const gpt2_handle* h, int* t);
int gpt2_set_step(gpt2_handle* h, int t);

/* ---------------------------------------------------------------- data */

/* Cuts one batch from a device stream of uint16 token ids [CH28 §28.3]:
 *   x[b,t] = stream[offset + b*T + t],  y[b,t] = stream[offset + b*T + t + 1]
 * for b < B, t < T (B*T+1 consecutive ids; every row is its own causal
 * window).  d_x, d_y are device int32 [B*T].  Needs offset >= 0 and
 * offset + B*T + 1 <= stream_len, else GPT2_ERR_ARG.  Bit-exact. */
int gpt2_batch_from_stream(gpt2_handle* h, const uint16_t* d_stream, int64_t stream_len,
                           int64_t offset, int B, int T, int32_t* d_x, int32_t* d_y);

/* ---------------------------------------------------------------- step */

/* Forward pass and mean loss [ZERO: autoregressive objective]:
 *   L = -1/(B*T) * sum_{b,t} log P(y[b,t] | x[b, 0..t])
 * x, y: int32 [B*T] ids in [0, vocab_size), device (tokens_on_device = 1) or
 * host (0; copied on the stream inside the call).  Saves the activations the
 * backward needs.  loss_out (host, nullable): when given the call
 * synchronises and writes L.  d_row_loss (device fp32 [B*T], nullable)
 * receives the per-position losses.  An id out of range is caught on the
 * device: the call (or the next synchronising call) returns GPT2_ERR_TOKEN
 * and the next gpt2_clip_adamw_step is refused.  Needs 1 <= B <= max_B,
 * 1 <= T <= max_Tseq. */
int gpt2_forward_loss(gpt2_handle* h, const int32_t* x, const int32_t* y, int B, int T,
                      int tokens_on_device, float* loss_out, float* d_row_loss);

/* Backward pass of the last gpt2_forward_loss: adds grad_scale * dL/dtheta
 * into the fp32 gradients (grad_scale = 1/accumulation steps for gradient
 * accumulation [LECTURE: gradient accumulation]).  The tied matrix receives
 * both the head and the embedding contributions.  GPT2_ERR_STATE if no
 * forward with saved activations precedes it. */
int gpt2_backward(gpt2_handle* h, float grad_scale);

/* Sets every gradient to zero (lazily: the next backward overwrites). */
int gpt2_zero_grad(gpt2_handle* h);

/* Global-norm clipping and AdamW over every parameter, one fused pass
 * [CS336 §2 AdamW, gradient clipping; ZERO: training loop]:
 *   n = sqrt(sum g^2);  s = min(1, max_norm / (n + 1e-6));  g' = s*g;  t += 1
 *   m = b1 m + (1-b1) g';  v = b2 v + (1-b2) g'^2
 *   p *= 1 - lr*wd (decay tensors only)
 *   p -= lr * sqrt(1-b2^t)/(1-b1^t) * m / (sqrt(v) + eps)
 * then refreshes the bf16 mirrors.  The stored gradients are read, not
 * rewritten.  grad_norm_out (host, nullable): the pre-clip n; when given the
 * call synchronises.  A non-finite n, or a token error in the forward, leaves
 * parameters, moments and t untouched (GPT2_ERR_NONFINITE / GPT2_ERR_TOKEN,
 * reported by this call when it synchronises, else by gpt2_synchronize). */
int gpt2_clip_adamw_step(gpt2_handle* h, float lr, float beta1, float beta2, float eps,
                         float weight_decay, float max_norm, float* grad_norm_out);

/* One whole step: zero_grad, forward_loss, backward(1), clip_adamw_step.
 * loss_out / grad_norm_out (host, nullable) as above. */
int gpt2_train_step(gpt2_handle* h, const int32_t* x, const int32_t* y, int B, int T,
                    int tokens_on_device, float lr, float beta1, float beta2, float eps,
                    float weight_decay, float max_norm, float* loss_out, float* grad_norm_out);

/* Kernel launches recorded into the step graph of gpt2_stream_begin (each
 * replay by gpt2_stream_steps runs exactly these); 0 when no step is
 * recorded.  Host only. */
int gpt2_stream_kernels(const gpt2_handle* h, int64_t* n);

/* Training on consecutive windows of a device-resident token stream, each
 * optimizer step replayed from a CUDA graph recorded once (no counterpart on
 * the pages, which launch every operation from Python; the step itself is
 * theirs: windows x = s[o .. o+BT), y = s[o+1 .. o+BT+1) [CH28 §28.3],
 * gradient accumulation over `accum` micro-batches with the loss scaled by
 * 1/accum [LECTURE], then norm, clip and AdamW [CS336 §2]).
 *
 * gpt2_stream_begin records one optimizer step: zero the gradients; accum
 * times { cut the B x T window at the device cursor, advance the cursor by
 * `stride` tokens, forward, backward with grad_scale 1/accum }; gradient
 * norm, clip to max_norm, AdamW (lr read on the device at replay).
 * d_stream: device uint16 ids [stream_len], must stay valid and unchanged in
 * size until gpt2_stream_end.  The cursor starts at `start` (for data
 * parallel rank r of R: start = r*B*T, stride = R*B*T).  A window that would
 * run past the stream is not read: the step's update is skipped and the next
 * status read (gpt2_stream_end, a loss or norm read) returns GPT2_ERR_ARG.
 * Profiling must be off.  Synchronises; nothing of the step runs yet.
 *
 * gpt2_stream_steps replays n_steps optimizer steps; lr: host [n_steps], the
 * learning rate of each (a schedule is computed by the caller).
 * Asynchronous on the handle's stream.
 *
 * gpt2_stream_end synchronises, writes the cursor (next window offset) to
 * *cursor_out (host, nullable), releases the graph and returns the device
 * status (GPT2_ERR_ARG for a window past the stream, GPT2_ERR_TOKEN,
 * GPT2_ERR_NONFINITE as in gpt2_clip_adamw_step).  The eager calls remain
 * usable before, between and after. */
int gpt2_stream_begin(gpt2_handle* h, const uint16_t* d_stream, int64_t stream_len, int64_t start,
                      int64_t stride, int B, int T, int accum, float beta1, float beta2, float eps,
                      float weight_decay, float max_norm);
int gpt2_stream_steps(gpt2_handle* h, int n_steps, const float* lr);
int gpt2_stream_end(gpt2_handle* h, int64_t* cursor_out);

/* Forward-only mean loss (no activations saved; the saved state of a
 * previous forward is invalidated) [CH28 §28.4: validation loss].  loss_out
 * (host) is required; the call synchronises. */
int gpt2_eval_loss(gpt2_handle* h, const int32_t* x, const int32_t* y, int B, int T,
                   int tokens_on_device, float* loss_out);

/* ---------------------------------------------------------------- generation */

/* Logits of the last position of every sequence [CS336: text generation,
 * "the last position's logits"; LECTURE: sampling loop]: the forward pass over
 * x (int32 [B*T], host or device as in gpt2_forward_loss; no activations
 * saved, a saved forward is invalidated), the final LayerNorm, and the tied
 * head for row T-1 of each sequence only:
 *   logits[b*ld + v] = hf[b, T-1] . wte[v]   for v < padded_vocab (fp32, device)
 * ld >= padded_vocab.  Synchronises (an id out of range gives GPT2_ERR_TOKEN).
 * Needs 1 <= B <= max_B, 1 <= T <= max_Tseq. */
int gpt2_logits_last(gpt2_handle* h, const int32_t* x, int B, int T, int tokens_on_device,
                     float* logits, int64_t ld);

/* Next token of each of B rows of fp32 logits [CS336: text generation —
 * temperature and top-p; LECTURE: top-k]:
 *   temperature == 0 or top_k == 1: the highest logit (the smaller id on ties);
 *   otherwise p_i = exp((z_i - max z) / temperature) in fp32 over the first V
 *   columns (the real vocabulary: padding columns are never drawn) and the
 *   weight of id i is the integer w_i = rint(p_i * 2^36), so every cumulative
 *   probability below is an exact integer sum; ids are ordered by p, the
 *   smaller id first among equal p; top_k > 0 keeps the first top_k of that
 *   order; top_p < 1 keeps its shortest prefix whose weight reaches top_p
 *   times the kept weight (the crossing id included); the draw walks the kept
 *   ids in increasing id order and returns the first id at which the running
 *   weight exceeds uniform[b] * (kept weight) (the last kept id if none does).
 * logits: device fp32, row b at logits + b*ld (ld >= V).  uniform: device fp32
 * [B] in [0, 1) (values outside are clamped; may be NULL for greedy choices).
 * out: device int32, out[b*out_stride].  Deterministic.  GPT2_ERR_ARG unless
 * 1 <= V <= 53248, B >= 1, temperature >= 0, top_k >= 0, 0 < top_p <= 1. */
int gpt2_sample(const float* logits, int64_t ld, int B, int V, float temperature, int top_k,
                float top_p, const float* uniform, int32_t* out, int64_t out_stride,
                void* stream);

/* Autoregressive generation without a KV cache [CS336: text generation —
 * every step recomputes the whole window, keeping only the most recent
 * context-length tokens]: out (device int32 [B, T0 + n_new]) receives the
 * prompt (device int32 [B, T0]) followed by n_new tokens; token T0 + s of row b
 * is gpt2_sample over the logits of gpt2_logits_last on the window
 * out[b, max(0, T0+s-W) .. T0+s) with W = min(max_T, max_Tseq), drawn with
 * uniform[s*B + b] (device fp32 [n_new, B]; NULL allowed for greedy choices).
 * Every step runs on the handle's stream without host synchronisation; the call
 * synchronises once at the end (GPT2_ERR_TOKEN for an id out of range in the
 * prompt).  No early stop at an end-of-text id: the caller cuts the rows.
 * Needs 1 <= B <= max_B, T0 >= 1, n_new >= 0, vocab_size <= 53248. */
int gpt2_generate(gpt2_handle* h, const int32_t* prompt, int B, int T0, int n_new,
                  float temperature, int top_k, float top_p, const float* uniform,
                  int32_t* out);

/* gpt2_generate with a key/value cache [CS336: text generation — the cache
 * reuses the history instead of recomputing the window]: the prompt runs once
 * through the model at positions 0 .. T0-1 and every layer's keys and values
 * are kept; each later step runs only the last generated token (position
 * T0+s-1) through the block, its attention reading the cached positions
 * 0 .. T0+s-1.  Same arguments, output and sampling as gpt2_generate, the same
 * tokens up to floating-point order (the same computation regrouped).  Needs
 * T0 + n_new <= min(max_T, max_Tseq) <= 4096 (no window slides) and a head
 * size dividing 128.  The first call allocates the cache: 2 * n_layer *
 * max_B * n_embd * min(max_T, max_Tseq) activation elements. */
int gpt2_generate_cached(gpt2_handle* h, const int32_t* prompt, int B, int T0, int n_new,
                         float temperature, int top_k, float top_p, const float* uniform,
                         int32_t* out);

/* Waits for the stream and reports a device-side error recorded since the
 * last check (token range, non-finite norm, bounded-wait timeout). */
int gpt2_synchronize(gpt2_handle* h);

/* Raw device address and length (elements) of one fp32 arena (GPT2_PARAM,
 * GPT2_GRAD, GPT2_ADAM_M, GPT2_ADAM_V).  The arena holds every tensor at its
 * own 64-element aligned offset (the padding stays 0), so it can be handed as
 * one buffer to a collective (e.g. a data-parallel gradient all-reduce) or a
 * checkpoint writer.  The pointer is owned by the handle.  Reading GPT2_GRAD
 * right after gpt2_zero_grad first materialises the zeros. */
int gpt2_arena(gpt2_handle* h, int which, float** ptr, int64_t* n_elems);

/* ---------------------------------------------------------------- data parallel */
/* The data-parallel step [LECTURE: DDP; CH28 §28.3, rank offsets]: every rank
 * runs forward and backward on its own windows, the ranks' gradients are
 * averaged (an all-reduce of the gradient arena), and every rank applies the
 * same clip + AdamW.  These calls let the caller overlap the exchange with
 * the backward pass: the arena is cut into buckets in the order the backward
 * finishes them, and the handle reports each one as it becomes final.  The
 * exchange itself is the caller's (e.g. NCCL through torch.distributed). */

/* Host-only layout of the arenas for configuration cfg (no handle, no device
 * call): tensor i (the order of gpt2_tensor_info) starts at element *offset
 * and holds *n_elems elements; its name is copied to name (name_len bytes,
 * NUL-terminated, nullable).  *n_tensors (nullable) receives the tensor count;
 * i = -1 asks for the count only. */
int gpt2_arena_layout(const gpt2_config* cfg, int i, char* name, int name_len, int64_t* offset,
                      int64_t* n_elems, int* n_tensors);

/* Host-only bucket plan of the gradient arena for configuration cfg, as
 * contiguous element ranges (offset[k], count[k]) each tagged with its bucket
 * bucket[k].  Bucket b < n_layer holds the four weight matrices of layer
 * n_layer-1-b (final once that layer's backward is done); bucket n_layer holds
 * wte, wpe and every vector (final after the embedding backward, the last
 * step of the backward).  The ranges cover the whole arena once, padding
 * included.  *n_ranges receives the number of ranges; the arrays are filled
 * only when max_ranges >= *n_ranges. */
int gpt2_grad_buckets(const gpt2_config* cfg, int max_ranges, int* n_ranges, int64_t* offset,
                      int64_t* count, int* bucket);

/* While fn is set (NULL clears it), gpt2_backward calls fn(user, b) on the
 * calling thread for b = 0 .. n_layer, in that order, each time right after it
 * has enqueued on the handle's stream the last work that writes bucket b: work
 * the callback enqueues on another stream after an event recorded on the
 * handle's stream at that moment sees bucket b final.  The callback must not
 * call into the handle.  It is not called while gpt2_stream_begin records a
 * step.  With gradient accumulation, set it before the last micro-batch's
 * backward only. */
typedef void (*gpt2_bucket_fn)(void* user, int bucket);
int gpt2_set_bucket_callback(gpt2_handle* h, gpt2_bucket_fn fn, void* user);

/* The exchange inside the library (NCCL, opened at run time): every rank
 * calls gpt2_dp_init with the same id (made by gpt2_dp_unique_id on one rank
 * and sent to the others, e.g. by torch.distributed) and its rank.  From then
 * on every backward that exchanges averages each gradient bucket over the
 * ranks as soon as it is final: an NCCL all-reduce (average) of the bucket's
 * ranges on the handle's communication stream, which first waits for the
 * handle's stream at that point; the handle's stream waits for the
 * communication stream at the end of the backward.  This includes the
 * backward recorded by gpt2_stream_begin, so one replayed graph holds a whole
 * data-parallel optimizer step (all ranks must replay the same number of
 * steps).  gpt2_dp_sync(h, 0) turns the exchange off for the backward calls
 * that follow (the micro-batches of an accumulation before the last one),
 * gpt2_dp_sync(h, 1) back on; gpt2_stream_begin exchanges on the last
 * micro-batch of each step only.  The communicator is destroyed by
 * gpt2_destroy (release every graph first, then destroy the handles, then
 * the caller's own process group).  GPT2_ERR_CUDA when NCCL cannot be
 * opened or fails. */
#define GPT2_DP_ID_BYTES 128
int gpt2_dp_unique_id(char* id);
int gpt2_dp_init(gpt2_handle* h, const char* id, int rank, int world);
int gpt2_dp_sync(gpt2_handle* h, int on);

/* ---------------------------------------------------------------- profiling */
/* Kernel groups timed by the built-in profiler. */
#define GPT2_PROF_GEMM 0        /* linear-layer contractions (fwd, dX, dW) */
#define GPT2_PROF_LMHEAD 1      /* tied-head contractions + cross-entropy rows */
#define GPT2_PROF_ATTN_FWD 2
#define GPT2_PROF_ATTN_BWD 3
#define GPT2_PROF_LN_FWD 4
#define GPT2_PROF_LN_BWD 5
#define GPT2_PROF_EMBED 6       /* embedding forward and backward */
#define GPT2_PROF_OPTIM 7       /* gradient norm + clip + AdamW */
#define GPT2_PROF_OTHER 8       /* column sums, copies, loss mean */
#define GPT2_PROF_NCAT 9

/* When enabled, every kernel group the handle launches is bracketed by CUDA
 * events on the handle's stream.  gpt2_profile_read synchronises and returns,
 * for group `cat` since the last reset: launches (kernels), summed device
 * time in ms, and the algorithmic FLOPs and HBM bytes of those launches
 * (nullable outputs).  cat = -1 returns the total launch count of the handle
 * (counted whether or not profiling is enabled). */
int gpt2_profile_enable(gpt2_handle* h, int enable);
int gpt2_profile_reset(gpt2_handle* h);
int gpt2_profile_read(gpt2_handle* h, int cat, int64_t* launches, double* ms, double* flops,
                      double* bytes);

/* ---------------------------------------------------------------- ops */

/* Tied LM head + mean cross-entropy alone [ZERO: output layer, fused
 * projection + cross-entropy; LECTURE: tied head over the padded vocabulary]:
 *   z = hidden W^T over all Vp rows; loss_m = logsumexp(z_m) - z_{m,y_m};
 *   *d_loss = mean_m loss_m;  dz = grad_scale/M * (softmax(z) - onehot(y))
 *   d_dh = dz W (overwritten), d_dw += dz^T hidden.
 * hidden: [M,C], W: [Vp,C] of type `dtype` (GPT2_BF16 or GPT2_F32), device.
 * y: device int32 [M] in [0, V).  d_loss: device fp32 [1].  d_lse (nullable):
 * device fp32 [M] log-normalisers.  d_dh (nullable, same type as hidden) and
 * d_dw (nullable, fp32 [Vp,C]) request the backward.  The [M,Vp] logits are
 * never stored: the forward reduces them tile by tile to per-row partials,
 * and the backward recomputes them chunk by chunk into one fixed-size dz
 * chunk buffer (2048 rows: 2048 x Vp bf16 = 206 MB at Vp = 50304 for
 * GPT2_BF16, fp32 for GPT2_F32), whatever M is.
 * workspace: device memory of at least gpt2_lmhead_ce_workspace() bytes.
 * C must be a multiple of 64 for GPT2_BF16.  Asynchronous on `stream`. */
int gpt2_lmhead_ce_workspace(int M, int C, int Vp, int dtype, size_t* bytes);
int gpt2_lmhead_ce(const void* hidden, const void* W, const int32_t* y, int M, int C, int Vp,
                   int V, int dtype, float grad_scale, float* d_loss, float* d_lse, void* d_dh,
                   float* d_dw, void* workspace, size_t workspace_bytes, void* stream);

/* LayerNorm forward over rows of x fp32 [M,C] (biased variance)
 * [ZERO: Transformer Block]:  y = gamma*(x-mu)*rstd + beta, written as
 * `y_dtype`; mean, rstd fp32 [M] (nullable).  Device buffers. */
int gpt2_layernorm_fwd(const float* x, const float* gamma, const float* beta, int64_t M, int C,
                       float eps, void* y, int y_dtype, float* mean, float* rstd, void* stream);

/* LayerNorm backward: with xh = (x-mu)*rstd, dxh = dy*gamma,
 *   dx += rstd*(dxh - mean(dxh) - xh*mean(dxh*xh)),
 *   dgamma += sum_m dy*xh, dbeta += sum_m dy   (deterministic column sums).
 * dy of type dy_dtype [M,C]; x, dx fp32 [M,C]; mean, rstd fp32 [M];
 * gamma, dgamma, dbeta fp32 [C].  workspace >= gpt2_layernorm_bwd_workspace(). */
int gpt2_layernorm_bwd_workspace(int64_t M, int C, size_t* bytes);
int gpt2_layernorm_bwd(const void* dy, int dy_dtype, const float* x, const float* mean,
                       const float* rstd, const float* gamma, int64_t M, int C, float* dx,
                       float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Causal multi-head attention [ZERO: Attention; LECTURE: causal attention]:
 * qkv [B,T,3C] (q | k | v, head h = channels [hD,(h+1)D)) of type `dtype`;
 * out [B,T,C] = per head softmax(q k^T / sqrt(D) with j > i excluded) v;
 * lse fp32 [B,H,T] = the softmax log-normaliser of each row (for the backward).
 * The [B,H,T,T] scores are never stored. */
int gpt2_attention_fwd(const void* qkv, int dtype, int B, int T, int C, int H, void* out,
                       float* lse, void* stream);

/* Backward of gpt2_attention_fwd: dqkv [B,T,3C] (overwritten) from dout
 * [B,T,C], qkv, out and lse of the forward.  workspace >=
 * gpt2_attention_bwd_workspace(), device memory owned by the caller: one
 * float per (batch, head, position) for Delta = rowsum(dO o O), and, for bf16
 * with head size 64, after it (at a 1 KB offset) the causal half of the score
 * gradients dS in bf16 (B*H*n(n+1)/2 tiles of 128 x 128, n = ceil(T/128);
 * 226 MB at B=16, T=1024, H=12), written by the dK/dV step and read by the dQ
 * step instead of recomputing them.  GPT2_ERR_ARG if the workspace is smaller. */
int gpt2_attention_bwd_workspace(int B, int T, int C, int H, int dtype, size_t* bytes);
int gpt2_attention_bwd(const void* dout, const void* qkv, const void* out, const float* lse,
                       int dtype, int B, int T, int C, int H, void* dqkv, void* workspace,
                       size_t workspace_bytes, void* stream);

/* gpt2_attention_bwd for callers that cannot allocate device memory: a
 * program that runs under a fixed memory budget already handed to another
 * allocator, or a loop that must not call cudaMalloc / cudaFree because those
 * calls can wait for the whole device to go idle.  Same arguments and the
 * same computation as gpt2_attention_bwd, but no workspace: the per-row
 * scratch lives in a fixed 4 MiB device array declared by the library (held
 * on every device that loads the library until the process exits), and the
 * dQ step recomputes the score gradients instead of keeping them (bf16 with
 * head size 64), so results can differ from gpt2_attention_bwd's in the last
 * bits.  No counterpart on the pages:
 * an interface variant only.
 *   - Limit: B*H*T <= 1,048,576 rows, else GPT2_ERR_ARG and a message.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *     The address is then kept for the rest of the process: resetting the
 *     device (cudaDeviceReset) or calling from a context other than the
 *     device's primary one is not supported.
 *   - Every call uses the same array, which keeps the last call's contents
 *     (each call writes what it reads first, so nothing needs clearing):
 *     calls that overlap on the GPU, e.g. on two streams, race. */
int gpt2_attention_bwd_noalloc(const void* dout, const void* qkv, const void* out,
                               const float* lse, int dtype, int B, int T, int C, int H,
                               void* dqkv, void* stream);

/* Dense contraction used by every linear layer (no counterpart on the pages
 * beyond "linear layer"; exported so it can be tested alone):
 *   D[m,n] = alpha * sum_k A(m,k) B(n,k)  (+ beta_accumulate * D[m,n] when
 *   accumulate = 1; D fp32 then)
 * A(m,k) = A[m*lda + k] when a_kmajor, else A[k*lda + m]; B likewise with ldb.
 * A, B of type `dtype`; D of type d_dtype (fp32, or bf16 when accumulate = 0).
 * workspace >= gpt2_matmul_workspace() (split-K partial sums). */
int gpt2_matmul_workspace(int M, int N, int K, size_t* bytes);
int gpt2_matmul(const void* A, int a_kmajor, int64_t lda, const void* B, int b_kmajor, int64_t ldb,
                int dtype, int M, int N, int K, float alpha, int accumulate, void* D, int d_dtype,
                int64_t ldd, void* workspace, size_t workspace_bytes, void* stream);

/* One linear layer of the block with its fused epilogue [ZERO: Transformer
 * Block; LECTURE: GELU (tanh form)], as the training step runs it:
 *   y = x W^T  with x [M,K] row-major and W [N,K] row-major (w_kn = 0: a
 *   layer's weight as it is stored), or y = x W with W [K,N] (w_kn = 1: the
 *   input-gradient contraction of the backward);
 * then, by `epi`:
 *   GPT2_LINEAR_BIAS       out = y + bias (bias may be NULL)
 *   GPT2_LINEAR_BIAS_GELU  out2 = y + bias rounded to `dtype` (the
 *                          pre-activation), out = GELU(out2); bias required
 *   GPT2_LINEAR_RESIDUAL   out = in + y + bias, in and out fp32 (the residual
 *                          stream; bias may be NULL; out must not overlap in)
 *   GPT2_LINEAR_GELU_BWD   out = y * GELU'(in), in = the pre-activation
 *                          (`dtype`); bias must be NULL
 * GELU(u) = u/2 (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))).  x, W and the
 * non-residual outputs are of type `dtype` (GPT2_BF16: tensor cores, fp32
 * accumulation; GPT2_F32: SIMT).  Rows are contiguous (strides K, N).
 * workspace >= gpt2_matmul_workspace(M, N, K).  GPT2_ERR_ARG on a null
 * required pointer, a size below 1 or an unknown epi. */
#define GPT2_LINEAR_BIAS 0
#define GPT2_LINEAR_BIAS_GELU 1
#define GPT2_LINEAR_RESIDUAL 2
#define GPT2_LINEAR_GELU_BWD 3
int gpt2_linear(int epi, const void* x, const void* w, int w_kn, const float* bias,
                const void* in, void* out, void* out2, int M, int N, int K, int dtype,
                void* workspace, size_t workspace_bytes, void* stream);

/* Self-check of the bounded device waits (no counterpart on the pages: the
 * failure handling of this library).  Every wait of the tensor-core kernels on
 * a barrier gives up after 2 s of device time, records a timeout (read back
 * as GPT2_ERR_TIMEOUT) and lets the kernel end.  This call runs one thread
 * that waits for a barrier phase nothing completes, synchronises the current
 * device (about 2 s), and sets *expired = 1 when the wait gave up and was
 * recorded, 0 otherwise; it clears the record afterwards, so the device and
 * the library stay usable.  Allocates 4 bytes with cudaMalloc. */
int gpt2_wait_selfcheck(int* expired);

/* Kernel launches the library has issued from the calling thread since the
 * process started, op-level calls and handle calls alike.  Kernels recorded
 * into a graph by gpt2_stream_begin count once, when recorded; replays by
 * gpt2_stream_steps are not counted here (gpt2_profile_read(h, -1) counts
 * them per handle). */
int gpt2_launch_count(int64_t* n);

/* Reads and clears the device error word shared by the op-level calls
 * (bounded-wait timeouts).  *code = GPT2_OK when nothing was recorded.
 * Synchronises the device. */
int gpt2_device_error(int* code);

#ifdef __cplusplus
}
#endif
#endif /* GPT2_B200_H */
