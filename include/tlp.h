/*
 * tlp.h — C ABI of the B200 (sm_100a) fused Transformer encoder layer,
 * forward and backward, pre-LN and post-LN.
 *
 * The layer computed is the BERT-style encoder layer of the "DeepSpeed
 * Transformer Kernel usage guide" (Step 1: one layer object per encoder
 * layer; Step 2: the configuration parameters batch_size, max_seq_length,
 * hidden_size, heads, attn_dropout_ratio, hidden_dropout_ratio,
 * pre_layer_norm, seed, fp16, intermediate_size, layer_norm_eps, training;
 * Step 3: the memory switches attn_dropout_checkpoint, normalize_invertible,
 * gelu_checkpoint), with the module order of "Forward-pass compute-graph
 * optimisation in the Transformer", section 2 (QKV projection, scaled
 * dot-product attention softmax(Q K^T / sqrt(d_k)) V, output projection,
 * residual + LayerNorm, FFN, residual + LayerNorm).
 *
 * Pre-LN:  h1 = LN1(x);  [Q|K|V] = h1 Wqkv^T + bqkv;
 *          ctx = dropout_a(softmax(Q K^T / sqrt(d) + mask)) V   (per head)
 *          x2 = x + dropout_h(ctx Wo^T + bo);  h2 = LN2(x2);
 *          y  = x2 + dropout_h(GELU(h2 W1^T + b1) W2^T + b2)
 * Post-LN: x2 = LN1(x + dropout_h(attn(x) Wo^T + bo));
 *          y  = LN2(x2 + dropout_h(FFN(x2)))
 * GELU is the erf form; LayerNorm is per token over the hidden axis with the
 * biased variance and eps inside the square root.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers on the device that was current
 *    when the layer's buffers were allocated; the caller owns them.
 *  - Tensors are dense row-major.  Activations are (batch, seq, hidden) =
 *    (T, H) with T = batch*seq.  Weights use the Linear convention
 *    [out_features, in_features]: wqkv (3H, H) with row blocks [Q; K; V] and
 *    head h owning rows h*d .. h*d+d-1 of each block; wo (H, H);
 *    w1 (F, H); w2 (H, F); biases and LayerNorm gamma/beta are vectors.
 *  - Activations and weights are in the layer's storage dtype (tl_dtype);
 *    the padding mask and every gradient of a weight are float32.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it; calls return before the GPU finishes.  Argument errors
 *    are reported synchronously and enqueue nothing.
 *  - Dropout draws its bits from Philox4x32-10 (Salmon et al., SC'11): the
 *    element with flat index e of dropout site s uses counter
 *    (e/8 mod 2^32, e/8 div 2^32, s, philox_offset) under key
 *    (seed mod 2^32, seed div 2^32); lane e mod 8 = k reads the 16-bit half
 *    (k mod 2) of output word (k div 2) and the element is kept when that
 *    lane is >= floor(p * 65536).  Kept values are scaled by 1/(1-p).
 *    Sites: 0 = attention probabilities, e = ((b*heads+h)*seq+i)*seq+j;
 *    1 = attention-block output, e = t*H+c; 2 = FFN output, e = t*H+c.
 */
#ifndef TLP_H
#define TLP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tl_layer tl_layer; /* opaque; owns saved activations + workspace */

typedef enum {
  TL_OK = 0,
  TL_EINVAL = 1,        /* bad argument; nothing was enqueued */
  TL_ENOMEM = 2,        /* device allocation failed */
  TL_ESTATE = 3,        /* call out of order (e.g. backward before a training forward) */
  TL_ECUDA = 4,         /* a CUDA call failed; see layer_last_error() */
  TL_ETIMEOUT = 5,      /* a bounded device-side wait gave up */
  TL_EUNSUPPORTED = 6   /* valid but not implemented for this configuration */
} tl_status;

typedef enum { TL_F32 = 0, TL_F16 = 1, TL_BF16 = 2 } tl_dtype;

/* Options ("DeepSpeed Transformer Kernel usage guide", Step 2 extra
 * parameters and Step 3 memory switches). */
typedef struct {
  int dtype;                     /* tl_dtype; default TL_F32 (fp16 = False) */
  float ln_eps;                  /* default 1e-12 */
  uint64_t philox_offset;        /* 4th Philox counter word; the layer id in a stack (default 0) */
  int gelu_checkpoint;           /* 1: keep only the FFN1 pre-activation U; GELU(U) and
                                    GELU'(U) are recomputed in backward (0: the forward
                                    keeps G = GELU(U) and GELU'(U)).  Results are bitwise
                                    identical. */
  int attn_dropout_checkpoint;   /* accepted; the attention kernels never store the
                                    dropped probabilities (only their keep bits, one bit
                                    per element), so this is always in effect */
  int normalize_invertible;      /* 1: LayerNorm backward from its output, the LayerNorm
                                    input is not needed (layer_backward may get x = NULL
                                    in pre-LN form); requires every gamma != 0 */
  int training;                  /* 1 (default): forward keeps what backward needs and applies
                                    dropout; 0: inference, dropout off, no backward */
  int gelu_tanh;                 /* 0 (default): GELU(u) = u * Phi(u), the erf form;
                                    1: the tanh approximation 0.5 u (1 + tanh(sqrt(2/pi)
                                    (u + 0.044715 u^3))) ("AI-infra engineers and the
                                    Transformer", section 2.3), forward and backward */
  int stochastic_mode;           /* 0 (default): every result is bitwise reproducible
                                    (column sums and split-K weight gradients are summed
                                    in a fixed order by a closing launch).  1: the
                                    backward adds them straight into the gradient
                                    outputs with float32 atomic adds, in arrival order,
                                    and skips that launch ("DeepSpeed Transformer Kernel
                                    usage guide", Step 2, stochastic_mode: a little
                                    faster, not reproducible).  Only the bias and
                                    LayerNorm gradients, and weight gradients whose K
                                    (= tokens) is split, may then differ from run to
                                    run, by float32 summation order; y, dx and every
                                    other gradient stay bitwise the same as with 0. */
} tl_options;

/* The twelve parameter tensors, all passed on every call (Step 2: the layer
 * hands all weights to the fused function at once).  Storage dtype. */
typedef struct {
  const void *wqkv, *bqkv, *wo, *bo, *ln1_g, *ln1_b;
  const void *w1, *b1, *w2, *b2, *ln2_g, *ln2_b;
} tl_weights;

/* Gradients of the twelve parameters, float32, same shapes as tl_weights.
 * Overwritten (not accumulated) by layer_backward. */
typedef struct {
  float *wqkv, *bqkv, *wo, *bo, *ln1_g, *ln1_b;
  float *w1, *b1, *w2, *b2, *ln2_g, *ln2_b;
} tl_grads;

/* Creates a layer.  ffn <= 0 means 4*hidden.  Rejected with TL_EINVAL:
 * non-positive sizes, hidden % heads != 0, head dim not in {16,32,64,128},
 * seq % 8 != 0, hidden % 8 != 0, ffn % 8 != 0, dropout ratios outside [0, 1).
 * No device memory is touched until layer_set_options or the first forward. */
tl_status layer_create(int batch, int seq, int hidden, int heads, int ffn,
                       float attn_dropout, float hidden_dropout, int pre_layer_norm,
                       uint64_t seed, tl_layer** out);

/* Fills *opt with the defaults listed in tl_options. */
void layer_default_options(tl_options* opt);

/* Sets the options and (re)allocates the layer's device buffers on the
 * current device (TL_ENOMEM on failure).  Must precede the first forward if
 * non-default options are wanted; afterwards it discards saved activations. */
tl_status layer_set_options(tl_layer* layer, const tl_options* opt);
tl_status layer_get_options(const tl_layer* layer, tl_options* opt);

/* Sets the dropout generator's key (seed, as given to layer_create) and 4th
 * counter word (tl_options.philox_offset) for the next forward, without
 * touching any buffer: a training loop gives each step masks of its own this
 * way (a stack, for instance, philox_offset = step * layers + layer).  A
 * backward always draws (or reads) the masks of the forward before it, so
 * calling this between the two is allowed.  TL_EINVAL for a NULL layer. */
tl_status layer_set_rng(tl_layer* layer, uint64_t seed, uint64_t philox_offset);

/* Forward.  x, y: (batch, seq, hidden) storage dtype; y must not alias x.
 * mask: NULL or (batch, seq) float32 additive key mask (0 for a valid key,
 * -inf for padding), broadcast over heads and queries.  A query row whose
 * keys are all masked gets zero attention output.  In training mode the
 * layer keeps what backward needs (it does not keep x: pass it again). */
tl_status layer_forward(tl_layer* layer, const void* x, const float* mask,
                        const tl_weights* w, void* y, void* stream);

/* Backward of the most recent training-mode forward (TL_ESTATE otherwise).
 * x: that forward's input (may be NULL only with normalize_invertible in
 * pre-LN form); dy: (batch, seq, hidden) upstream gradient; dx receives the
 * input gradient; g receives every parameter gradient (float32, overwritten).
 * The mask of that forward is reused and must still be valid. */
tl_status layer_backward(tl_layer* layer, const void* x, const void* dy,
                         const tl_weights* w, tl_grads* g, void* dx, void* stream);

/* Device bytes the layer holds: its saved activations, plus its own scratch
 * unless it uses a shared one (layer_share_scratch). */
size_t layer_workspace_bytes(const tl_layer* layer);

/* Scratch sharing ("DeepSpeed Transformer Kernel usage guide", Step 3: the
 * memory switches exist so that larger micro-batches fit).  A layer's
 * scratch holds what lives only within one layer_forward or layer_backward
 * call (the backward's intermediate gradients, GELU(U) between the two FFN
 * GEMMs in recompute mode, column-sum partials, split-K partials); nothing
 * in it is needed from one call to the next.  Layers of a stack that never
 * run at the same time can therefore share one scratch.
 * layer_scratch_bytes: the size this layer's scratch needs (its options
 * included).  layer_share_scratch: the layer frees its own scratch and uses
 * `scratch` (a device buffer of `bytes` >= layer_scratch_bytes, 256-byte
 * aligned, owned by the caller and valid for the layer's lifetime) instead;
 * TL_EINVAL if it is null, unaligned or too small.  Calls of layers that
 * share a scratch must not overlap on the GPU (enqueue them on one stream,
 * or order the streams).  layer_set_options keeps a shared scratch while it
 * is large enough for the new options, else the layer allocates its own. */
size_t layer_scratch_bytes(const tl_layer* layer);
tl_status layer_share_scratch(tl_layer* layer, void* scratch, size_t bytes);

/* Text of the last error on this layer ("" if none).  Valid until the next call. */
const char* layer_last_error(const tl_layer* layer);

/* Releases every device buffer of the layer.  Synchronises the device first. */
void layer_destroy(tl_layer* layer);

/* Test hook: writes keep[i] = 1 if flat element e0+i of `site` is kept under
 * the Philox contract above, else 0, for i < n (device buffer of n bytes).
 * e0 and n must be multiples of 8.  Uses the same device code as the layer. */
tl_status tl_dropout_keep_mask(uint64_t seed, uint64_t philox_offset, int site, float p,
                               uint64_t e0, uint64_t n, uint8_t* keep, void* stream);

/* Test hook: g[i] = GELU(u[i]) and dg[i] = GELU'(u[i]) for i < n (float32
 * device buffers), evaluated by the same device code the layer's GEMM
 * epilogues use: erf form, Phi(u) from the normal-tail approximation of
 * Abramowitz & Stegun 26.2.17 (absolute error below 7.5e-8) in float32. */
tl_status tl_gelu_eval(const float* u, float* g, float* dg, uint64_t n, void* stream);

/* Test hook: as tl_gelu_eval for the tanh form (tl_options.gelu_tanh), the
 * same device code as the layer's epilogues with that option. */
tl_status tl_gelu_tanh_eval(const float* u, float* g, float* dg, uint64_t n, void* stream);

/* Waits for all work on the current device, then reports TL_ECUDA if a CUDA
 * error is pending, TL_ETIMEOUT if a bounded device-side wait of a
 * tensor-core kernel gave up since the last call (the flag is cleared), else
 * TL_OK.  Blocks the host. */
tl_status tl_device_check(void);

/* Failure detection.  Every wait of the tensor-core and row kernels on an
 * mbarrier (for a copy, an MMA or another warp) is bounded: once it has
 * waited longer than the limit it records an error, lets the copies it has
 * issued land, frees its tensor memory and returns, and tl_device_check
 * reports TL_ETIMEOUT.  tl_set_wait_limit_ns sets that limit for the
 * current device (ns; 0 restores the default of 2 s); it is synchronous
 * and applies to launches enqueued after it.  A limit shorter than the
 * longest legitimate wait (microseconds in these kernels) makes healthy
 * kernels give up.
 * tl_wait_probe enqueues a one-thread kernel whose single bounded wait
 * nothing ever satisfies: it gives up after the current limit with nothing
 * else in flight, so the next tl_device_check reports TL_ETIMEOUT and the
 * context stays usable (a test of the detection path). */
tl_status tl_set_wait_limit_ns(uint64_t ns);
tl_status tl_wait_probe(void* stream);

/* Profiling (off by default).  While enabled, the library brackets each of
 * its kernel launches with a pair of CUDA events on the launching stream.
 * tl_profile_read synchronises the device, fills ms[c] (summed elapsed
 * milliseconds) and launches[c] (bracketed launch groups) for each class c <
 * n accumulated since the previous read, clears them, and returns the number
 * of classes: 0 GEMM, 1 attention forward, 2 attention backward,
 * 3 LayerNorm forward, 4 LayerNorm backward, 5 other bandwidth kernels. */
void tl_profile_enable(int on);
int tl_profile_read(double* ms, long long* launches, int n);

/* Total number of kernels the library has launched since it was loaded. */
long long tl_launch_count(void);

/* Column sums that allocate nothing: db[c] = sum over r < rows of dz[r, c]
 * (dz row-major (rows, cols) in storage dtype `dtype`, db float32 (cols)),
 * the bias gradient of a Linear layer whose output gradient is dz.  The
 * source pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory (memory owned by a framework's caching
 * allocator or a fixed budget, or code running inside a global-mode stream
 * capture, where cudaMalloc is not allowed).
 * Scratch: a 2 MiB array in the library's device memory, held by every GPU
 * that loads the library until the process exits.  Limits: cols <= 8192 and a
 * multiple of 8, rows >= 1, both pointers 16-byte aligned, else TL_EINVAL.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * The address is kept per device together with the CUDA context it belongs
 * to; after a device reset (a new context) the next call looks it up again
 * and, like a first call, belongs before any capture.
 * Every call shares the one array and overwrites it: calls that overlap on
 * the GPU (other streams, other threads) race and must be serialised by the
 * caller.  Enqueued on `stream` (a cudaStream_t); returns before the GPU
 * finishes.  TL_ECUDA if a CUDA call fails, including an error that an
 * earlier call left pending when this one starts (it is cleared). */
tl_status tl_bias_grad_noalloc(int dtype, const void* dz, int rows, int cols, float* db, void* stream);

/* Progressive Layer Dropping for a stack of layers ("Progressive Layer
 * Dropping" page, schedule section).  Host functions; no device work.
 *
 * tl_pld_theta: the keep level at global step `step`,
 *   theta(t) = (1 - theta_bar) * exp(-gamma * t) + theta_bar,
 * which is 1 at t = 0 and tends to theta_bar.
 * tl_pld_keep_prob: probability that layer `layer` (0-based) of
 * `num_layers` runs at keep level theta: 1 - (layer+1)/num_layers * (1-theta)
 * (the depth profile is linear; the last layer is kept with probability
 * theta).  -1 for a layer index outside [0, num_layers).
 * tl_pld_keep: 1 if the layer runs at this step, 0 if it is skipped (the
 * identity in forward and backward), -1 for a bad layer index.  Decided by
 * Philox4x32-10 with counter (step mod 2^32, step div 2^32, 3, layer) and key
 * (seed mod 2^32, seed div 2^32): kept when output word 0 < floor(p * 2^32),
 * p the keep probability (always kept when p >= 1, never when p <= 0).
 * Equal seeds and steps give equal decisions on every rank. */
double tl_pld_theta(double theta_bar, double gamma, uint64_t step);
double tl_pld_keep_prob(int layer, int num_layers, double theta);
int tl_pld_keep(uint64_t seed, uint64_t step, int layer, int num_layers, double theta);

const char* tl_status_string(tl_status s);

#ifdef __cplusplus
}
#endif

#endif /* TLP_H */
