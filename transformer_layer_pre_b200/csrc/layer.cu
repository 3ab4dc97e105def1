// layer.cu — the C ABI (include/tlp.h): layer handle, buffers and the
// forward/backward schedules of the encoder layer.
//
// Schedules (T tokens, storage type of the layer):
//  pre-LN forward   LN1 -> QKV GEMM (+bias, head split) -> attention ->
//                   out-proj GEMM (+bias, dropout, +x) -> LN2 ->
//                   FFN1 GEMM (+bias, GELU) -> FFN2 GEMM (+bias, dropout, +x2)
//  pre-LN backward  dropout'(dY) + db2 -> dW2, dU = (dZ2 W2) GELU'(U) -> db1,
//                   dW1, dH2 -> LN2' (+dY, dropout' -> dA, dbo) -> dWo, dctx ->
//                   attention' -> dbqkv, dWqkv, dH1 -> LN1' (+dx2) = dx
//  post-LN          the same kernels wired per "Forward-pass compute-graph
//                   optimisation in the Transformer", section 2 (residual add
//                   then LayerNorm after each block).
// Bias gradients are column sums of the stored output gradient of their
// Linear; weight gradients are float32 GEMMs over the tokens.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/tlp.h"
#include "kernels.h"
#include "profile.h"

namespace tlp {
bool rowwise_supports_hidden(int H);
void attn_simt_fwd_run(int dt, const AttnArgs& a, cudaStream_t s);
void attn_simt_bwd_run(int dt, const AttnArgs& a, cudaStream_t s);
void attn_tc_fwd_run(int dt, const AttnArgs& a, cudaStream_t s);
void attn_tc_bwd_run(int dt, const AttnArgs& a, cudaStream_t s);
bool attn_tc_supports(int dt, const AttnArgs& a);
bool attn_tc_fuses_colsum(int dt, const AttnArgs& a);
}  // namespace tlp

using namespace tlp;

struct tl_layer {
  int B, S, H, nh, d, F, T;
  float pa, ph;
  int pre_ln;
  uint64_t seed;
  tl_options opt;
  // Philox key and 4th counter word of the current (or last training)
  // forward: its backward uses them even if layer_set_rng changed seed and
  // opt.philox_offset since
  uint64_t drop_seed = 0, drop_offset = 0;
  int device = -1;
  char* arena = nullptr;          // saved activations (forward -> backward)
  size_t arena_bytes = 0;
  char* scratch = nullptr;        // scratch of one call: the layer's own, or the caller's
  size_t scratch_bytes = 0;
  bool scratch_owned = false;
  bool have_fwd = false;
  const float* mask = nullptr;
  std::string err;

  // saved activations
  void *h1 = nullptr, *qkv = nullptr, *ctx = nullptr, *x2 = nullptr, *h2 = nullptr;
  void *u = nullptr, *g = nullptr, *res1 = nullptr, *res2 = nullptr, *yout = nullptr;
  float *mean1 = nullptr, *rstd1 = nullptr, *mean2 = nullptr, *rstd2 = nullptr, *lse = nullptr;
  // backward scratch
  void *big = nullptr;     // (T, F): G recompute / dU
  void *dz2 = nullptr, *dh = nullptr, *dx2 = nullptr, *da = nullptr, *dctx = nullptr, *dres = nullptr;
  void *dqkv = nullptr;
  float *dvec = nullptr, *part = nullptr;
  size_t part_floats = 0;
  // hidden-dropout keep bits of sites 1 and 2 (one byte per 8 elements)
  uint8_t *keep1 = nullptr, *keep2 = nullptr;
  // attention dropout keep bits (site 0), written by the forward for the
  // backward: [B*nh][128][16] bytes for S <= 128, else [B*nh][S][S/8]; or null
  uint8_t* akeep = nullptr;
  // per sequence: one past its last unmasked key (filled by the long-sequence forward)
  int* kv_ext = nullptr;
  // split-K scratch of the four weight gradients (W2, W1, Wo, Wqkv), each its
  // own, so every split sum can wait for the closing finalize launch
  float* splitk[4] = {nullptr, nullptr, nullptr, nullptr};
  size_t splitk_floats[4] = {0, 0, 0, 0};
  int gemm_err = 0;
};

namespace {

tl_status fail(tl_layer* L, tl_status st, const char* msg) {
  if (L) L->err = msg;
  return st;
}

tl_status check_cuda(tl_layer* L, const char* where) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    if (L) L->err = std::string(where) + ": " + cudaGetErrorString(e);
    return TL_ECUDA;
  }
  return TL_OK;
}

DropoutParams make_drop(const tl_layer* L, float p) {
  DropoutParams d;
  d.seed = L->drop_seed;
  d.offset = L->drop_offset;
  const bool on = L->opt.training && p > 0.0f;
  d.thr = on ? (uint32_t)std::floor((double)p * 65536.0) : 0u;
  d.scale = on ? 1.0f / (1.0f - p) : 1.0f;
  return d;
}

void free_scratch(tl_layer* L) {
  if (L->scratch && L->scratch_owned) {
    cudaDeviceSynchronize();
    cudaFree(L->scratch);
  }
  L->scratch = nullptr;
  L->scratch_bytes = 0;
  L->scratch_owned = false;
}

void free_buffers(tl_layer* L) {
  if (L->arena) {
    cudaDeviceSynchronize();
    cudaFree(L->arena);
  }
  L->arena = nullptr;
  L->arena_bytes = 0;
  free_scratch(L);
  L->have_fwd = false;
}

struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(char* b) : base(b) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  }
};

// Lays out the buffers that live from a forward to its backward; with
// base == nullptr it only measures.
size_t carve(tl_layer* L, char* base) {
  Carver c(base);
  const size_t es = dtype_size(L->opt.dtype);
  const size_t TH = (size_t)L->T * L->H, TF = (size_t)L->T * L->F;
  const bool ckpt = L->opt.gelu_checkpoint != 0;
  L->qkv = c.take(3 * TH * es);
  L->ctx = c.take(TH * es);
  L->lse = (float*)c.take((size_t)L->B * L->nh * L->S * 4);
  L->mean1 = (float*)c.take((size_t)L->T * 4);
  L->rstd1 = (float*)c.take((size_t)L->T * 4);
  L->mean2 = (float*)c.take((size_t)L->T * 4);
  L->rstd2 = (float*)c.take((size_t)L->T * 4);
  L->x2 = c.take(TH * es);
  // u: the FFN1 output U when G is recomputed in backward (checkpoint mode),
  // else GELU'(U), written by the FFN1 epilogue next to G so that the
  // backward's dU needs no special function
  L->u = c.take(TF * es);
  if (!ckpt) L->g = c.take(TF * es);   // recompute mode: G lives in the scratch's `big` (carve_scratch)
  if (L->pre_ln) {
    L->h1 = c.take(TH * es);
    L->h2 = c.take(TH * es);
    L->res1 = L->res2 = L->yout = nullptr;
  } else {
    L->h1 = L->h2 = nullptr;
    L->res1 = L->opt.normalize_invertible ? nullptr : c.take(TH * es);
    L->res2 = L->opt.normalize_invertible ? nullptr : c.take(TH * es);
    L->yout = L->opt.normalize_invertible ? c.take(TH * es) : nullptr;
  }
  L->keep1 = (uint8_t*)c.take((size_t)L->T * L->H / 8);
  L->keep2 = (uint8_t*)c.take((size_t)L->T * L->H / 8);
  // attention keep bits (site 0), one bit per element: [B*nh][128][16] bytes
  // for S <= 128, the flat [B*nh][S][S/8] otherwise
  const size_t akeep_bytes = L->S <= 128 ? (size_t)L->B * L->nh * 128 * 16 : (size_t)L->B * L->nh * L->S * (L->S / 8);
  L->akeep = L->pa > 0.0f ? (uint8_t*)c.take(akeep_bytes) : nullptr;
  L->kv_ext = (int*)c.take((size_t)L->B * 4);
  return c.off;
}

// Lays out the scratch of one call (nothing in it outlives a forward or a
// backward: layers that never run at the same time may share it); with
// base == nullptr it only measures.
size_t carve_scratch(tl_layer* L, char* base) {
  Carver c(base);
  const size_t es = dtype_size(L->opt.dtype);
  const size_t TH = (size_t)L->T * L->H, TF = (size_t)L->T * L->F;
  // (T, F): dU in backward; in recompute mode also G, from FFN1 to FFN2 in
  // the forward and recomputed from U in the backward
  L->big = c.take(TF * es);
  if (L->opt.gelu_checkpoint) L->g = L->big;
  L->dz2 = c.take(TH * es);
  L->dh = c.take(TH * es);
  L->dx2 = c.take(TH * es);
  L->da = c.take(TH * es);
  L->dctx = c.take(TH * es);
  L->dres = c.take(TH * es);
  L->dqkv = c.take(3 * TH * es);
  L->dvec = (float*)c.take((size_t)L->B * L->nh * L->S * 4);
  const int np = std::max(std::max(std::max(ln_bwd_parts(L->T), rowdrop_parts(L->T)), colsum_parts(L->T)),
                          std::max((L->T + 255) / 256 * 8, L->B * 4));   // + partial rows of fused column sums
  const int maxc = std::max(3 * L->H, L->F);
  L->part_floats = (size_t)np * maxc;
  L->part = (float*)c.take((size_t)kMaxFinalize * L->part_floats * 4);   // one slot per parameter column sum
  const int dt = L->opt.dtype, T = L->T, H = L->H, F = L->F;
  const size_t wsf[4] = {gemm_splitk_ws_floats(dt, H, F, T), gemm_splitk_ws_floats(dt, F, H, T),
                         gemm_splitk_ws_floats(dt, H, H, T), gemm_splitk_ws_floats(dt, 3 * H, H, T)};
  for (int i = 0; i < 4; ++i) {
    L->splitk_floats[i] = wsf[i];
    L->splitk[i] = wsf[i] ? (float*)c.take(wsf[i] * 4) : nullptr;
  }
  return c.off;
}

// Bytes of the scratch (measured on a copy: measuring lays out null pointers).
size_t scratch_size(const tl_layer* L) {
  tl_layer tmp = *L;
  return carve_scratch(&tmp, nullptr);
}

tl_status ensure_buffers(tl_layer* L) {
  if (L->arena && L->scratch) {
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != L->device) return fail(L, TL_EINVAL, "layer used on a different device than it was allocated on");
    return TL_OK;
  }
  if (!L->arena) {
    const size_t bytes = carve(L, nullptr);
    cudaGetDevice(&L->device);
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return fail(L, TL_ENOMEM, "cudaMalloc of the layer workspace failed");
    }
    L->arena = (char*)p;
    L->arena_bytes = bytes;
    carve(L, L->arena);
  }
  if (!L->scratch) {
    const size_t bytes = carve_scratch(L, nullptr);
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return fail(L, TL_ENOMEM, "cudaMalloc of the layer scratch failed");
    }
    L->scratch = (char*)p;
    L->scratch_bytes = bytes;
    L->scratch_owned = true;
    carve_scratch(L, L->scratch);
  }
  return TL_OK;
}

// A GEMM whose B is a weight: never the output of the kernel before it, so
// the tensor-core kernel may load B before it waits for that kernel.
GemmDesc gdesc(tl_layer* L, int M, int N, int K, const void* A, int lda, bool ak, const void* B, int ldb, bool bk) {
  GemmDesc g{M, N, K, A, lda, ak, B, ldb, bk, nullptr, 0};
  g.b_early = true;
  return g;
}

// A weight-gradient GEMM (float32 out) with split-K scratch `which` (0 W2,
// 1 W1, 2 Wo, 3 Wqkv) whose split sum joins the closing finalize list.  Its
// B is an activation the forward saved (G, the FFN input, ctx, the
// attention input), not the output of the kernel before it, unless the
// caller says otherwise (b_early = false).
GemmDesc wdesc(tl_layer* L, int which, FinalizeList* fin, int M, int N, int K, const void* A, int lda, const void* B,
               int ldb) {
  GemmDesc g{M, N, K, A, lda, false, B, ldb, false, L->splitk[which], L->splitk_floats[which]};
  g.defer = fin;
  g.b_early = true;
  return g;
}

void gemm(tl_layer* L, int M, int N, int K, const void* A, int lda, bool ak, const void* B, int ldb, bool bk,
          const EpiParams& e, cudaStream_t s) {
  const GemmDesc g = gdesc(L, M, N, K, A, lda, ak, B, ldb, bk);
  ProfScope p_(PC_GEMM, s);
  if (gemm_run(L->opt.dtype, g, e, s) != 0) L->gemm_err = 1;
}

// A weight gradient and an input gradient that read the same operand, in one
// launch (they must not write what the other reads).
void gemm2(tl_layer* L, const GemmDesc& ga, const EpiParams& ea, const GemmDesc& gb, const EpiParams& eb,
           cudaStream_t s) {
  ProfScope p_(PC_GEMM, s);
  if (gemm_run2(L->opt.dtype, ga, ea, gb, eb, s) != 0) L->gemm_err = 1;
}

// Tensor pointers must be 16-byte aligned (vector loads and TMA).
bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

EpiParams epi(int kind, void* out, int ldo) {
  EpiParams e;
  std::memset(&e, 0, sizeof(e));
  e.kind = kind;
  e.out = out;
  e.ldo = ldo;
  return e;
}

// Column partial sums of a (T, cols) stored matrix into partial slot `slot`,
// summed into `out` by the backward's closing finalize (stochastic mode:
// added into `out`, which holds zeros, with atomics).
void bias_grad(tl_layer* L, const void* X, int cols, int slot, float* out, FinalizeList& fin, cudaStream_t s) {
  ProfScope p_(PC_ROWWISE, s);
  if (L->opt.stochastic_mode) {
    colsum_run(L->opt.dtype, X, L->T, cols, out, s, 1);
    return;
  }
  float* part = L->part + (size_t)slot * L->part_floats;
  colsum_run(L->opt.dtype, X, L->T, cols, part, s);
  fin.job[fin.n++] = {part, out, colsum_parts(L->T), cols};
}

void attn_fwd(tl_layer* L, const AttnArgs& a, cudaStream_t s) {
  ProfScope p_(PC_ATTN_FWD, s);
  if (attn_tc_supports(L->opt.dtype, a)) attn_tc_fwd_run(L->opt.dtype, a, s);
  else attn_simt_fwd_run(L->opt.dtype, a, s);
}
void attn_bwd(tl_layer* L, const AttnArgs& a, cudaStream_t s) {
  ProfScope p_(PC_ATTN_BWD, s);
  if (attn_tc_supports(L->opt.dtype, a)) attn_tc_bwd_run(L->opt.dtype, a, s);
  else attn_simt_bwd_run(L->opt.dtype, a, s);
}

AttnArgs attn_args(tl_layer* L, const float* mask) {
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  const size_t es = dtype_size(L->opt.dtype);
  const size_t TH = (size_t)L->T * L->H;
  a.B = L->B; a.S = L->S; a.nh = L->nh; a.d = L->d;
  a.q = L->qkv;
  a.k = (char*)L->qkv + TH * es;
  a.v = (char*)L->qkv + 2 * TH * es;
  a.mask = mask;
  a.scale = (float)(1.0 / std::sqrt((double)L->d));
  a.drop = make_drop(L, L->pa);
  a.ctx = L->ctx;
  a.lse = L->lse;
  a.dctx = L->dctx;
  a.dvec = L->dvec;
  a.dqkv = L->dqkv;
  a.keep = L->akeep;
  a.kv_ext = L->kv_ext;
  return a;
}

}  // namespace

extern "C" {

const char* tl_status_string(tl_status s) {
  switch (s) {
    case TL_OK: return "ok";
    case TL_EINVAL: return "invalid argument";
    case TL_ENOMEM: return "out of device memory";
    case TL_ESTATE: return "call out of order";
    case TL_ECUDA: return "CUDA error";
    case TL_ETIMEOUT: return "device wait timed out";
    case TL_EUNSUPPORTED: return "unsupported configuration";
  }
  return "unknown status";
}

void layer_default_options(tl_options* o) {
  if (!o) return;
  std::memset(o, 0, sizeof(*o));
  o->dtype = TL_F32;
  o->ln_eps = 1e-12f;
  o->philox_offset = 0;
  o->training = 1;
}

tl_status layer_create(int batch, int seq, int hidden, int heads, int ffn, float attn_dropout, float hidden_dropout,
                       int pre_layer_norm, uint64_t seed, tl_layer** out) {
  if (!out) return TL_EINVAL;
  *out = nullptr;
  if (batch <= 0 || seq <= 0 || hidden <= 0 || heads <= 0) return TL_EINVAL;
  if (hidden % heads != 0) return TL_EINVAL;
  const int d = hidden / heads;
  if (d != 16 && d != 32 && d != 64 && d != 128) return TL_EINVAL;
  if (seq % 8 != 0 || hidden % 8 != 0) return TL_EINVAL;
  const int F = ffn <= 0 ? 4 * hidden : ffn;
  if (F % 8 != 0) return TL_EINVAL;
  if (!(attn_dropout >= 0.0f && attn_dropout < 1.0f) || !(hidden_dropout >= 0.0f && hidden_dropout < 1.0f))
    return TL_EINVAL;
  if (!rowwise_supports_hidden(hidden)) return TL_EUNSUPPORTED;
  if ((long long)batch * seq > (1LL << 30)) return TL_EUNSUPPORTED;
  tl_layer* L = new (std::nothrow) tl_layer();
  if (!L) return TL_ENOMEM;
  L->B = batch; L->S = seq; L->H = hidden; L->nh = heads; L->d = d; L->F = F; L->T = batch * seq;
  L->pa = attn_dropout; L->ph = hidden_dropout;
  L->pre_ln = pre_layer_norm ? 1 : 0;
  L->seed = seed;
  layer_default_options(&L->opt);
  *out = L;
  return TL_OK;
}

tl_status layer_set_options(tl_layer* L, const tl_options* o) {
  if (!L || !o) return TL_EINVAL;
  if (o->dtype < TL_F32 || o->dtype > TL_BF16) return fail(L, TL_EINVAL, "unknown dtype");
  if (!(o->ln_eps > 0.0f)) return fail(L, TL_EINVAL, "ln_eps must be positive");
  // shared scratch stays shared if it still fits the new options
  char* shared = (L->scratch && !L->scratch_owned) ? L->scratch : nullptr;
  const size_t shared_bytes = shared ? L->scratch_bytes : 0;
  free_buffers(L);
  L->opt = *o;
  L->opt.training = o->training ? 1 : 0;
  L->opt.gelu_tanh = o->gelu_tanh ? 1 : 0;
  L->opt.stochastic_mode = o->stochastic_mode ? 1 : 0;
  if (shared && shared_bytes >= scratch_size(L)) {
    L->scratch = shared;
    L->scratch_bytes = shared_bytes;
    L->scratch_owned = false;
    carve_scratch(L, L->scratch);
  }
  return ensure_buffers(L);
}

tl_status layer_set_rng(tl_layer* L, uint64_t seed, uint64_t philox_offset) {
  if (!L) return TL_EINVAL;
  L->seed = seed;
  L->opt.philox_offset = philox_offset;
  return TL_OK;
}

tl_status layer_get_options(const tl_layer* L, tl_options* o) {
  if (!L || !o) return TL_EINVAL;
  *o = L->opt;
  return TL_OK;
}

size_t layer_workspace_bytes(const tl_layer* L) {
  return L ? L->arena_bytes + (L->scratch_owned ? L->scratch_bytes : 0) : 0;
}

size_t layer_scratch_bytes(const tl_layer* L) { return L ? scratch_size(L) : 0; }

tl_status layer_share_scratch(tl_layer* L, void* scratch, size_t bytes) {
  if (!L) return TL_EINVAL;
  L->err.clear();
  if (!scratch) return fail(L, TL_EINVAL, "null scratch pointer");
  if (reinterpret_cast<uintptr_t>(scratch) & 255) return fail(L, TL_EINVAL, "scratch must be 256-byte aligned");
  const size_t need = scratch_size(L);
  if (bytes < need) return fail(L, TL_EINVAL, "scratch smaller than layer_scratch_bytes");
  free_scratch(L);
  L->scratch = (char*)scratch;
  L->scratch_bytes = bytes;
  L->scratch_owned = false;
  carve_scratch(L, L->scratch);
  return TL_OK;
}

const char* layer_last_error(const tl_layer* L) { return L ? L->err.c_str() : "null layer"; }

void layer_destroy(tl_layer* L) {
  if (!L) return;
  free_buffers(L);
  delete L;
}

static bool weights_ok(const tl_weights* w) {
  return w && w->wqkv && w->bqkv && w->wo && w->bo && w->ln1_g && w->ln1_b && w->w1 && w->b1 && w->w2 && w->b2 &&
         w->ln2_g && w->ln2_b;
}

tl_status layer_forward(tl_layer* L, const void* x, const float* mask, const tl_weights* w, void* y, void* stream) {
  if (!L) return TL_EINVAL;
  L->err.clear();
  if (!x || !y || !weights_ok(w)) return fail(L, TL_EINVAL, "null tensor pointer");
  if (x == y) return fail(L, TL_EINVAL, "y must not alias x");
  if (!aligned(x) || !aligned(y) || !aligned(w->wqkv) || !aligned(w->wo) || !aligned(w->w1) || !aligned(w->w2) ||
      !aligned(w->bqkv) || !aligned(w->bo) || !aligned(w->b1) || !aligned(w->b2) || !aligned(w->ln1_g) ||
      !aligned(w->ln1_b) || !aligned(w->ln2_g) || !aligned(w->ln2_b))
    return fail(L, TL_EINVAL, "tensor pointers must be 16-byte aligned");
  tl_status st = ensure_buffers(L);
  if (st != TL_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int dt = L->opt.dtype, T = L->T, H = L->H, F = L->F;
  const bool train = L->opt.training != 0;
  L->have_fwd = false;
  L->drop_seed = L->seed;
  L->drop_offset = L->opt.philox_offset;

  EpiParams eq = epi(EPI_QKV, L->qkv, 3 * H);
  eq.bias = w->bqkv; eq.seq = L->S; eq.hidden = H; eq.head_dim = L->d; eq.heads = L->nh; eq.tokens = T;
  AttnArgs aa = attn_args(L, mask);

  EpiParams eo = epi(EPI_BIAS_DROP_RES, nullptr, H);
  eo.bias = w->bo; eo.res = x; eo.drop = make_drop(L, L->ph); eo.site = 1;
  EpiParams e1 = epi(L->opt.gelu_checkpoint ? EPI_BIAS_GELU : EPI_BIAS_GELU_D, L->u, F);
  e1.bias = w->b1; e1.out2 = L->g; e1.gelu_tanh = L->opt.gelu_tanh ? 1 : 0;
  EpiParams e2 = epi(EPI_BIAS_DROP_RES, nullptr, H);
  e2.bias = w->b2; e2.drop = make_drop(L, L->ph); e2.site = 2;

  // hidden-dropout keep bits are drawn once, ahead of their consumers, which
  // read them instead of drawing Philox: both sites by the QKV GEMM's CTA
  // pairs that sit out its last round; where it has none (small batches), by
  // the LayerNorm forward before the consumer (pre-LN: LN1 for site 1, LN2 for
  // site 2; post-LN: LN1 for site 2)
  const bool keepbits = eo.drop.thr != 0;
  const bool k1_gemm = keepbits && gemm_tc_bubble_pairs(dt, T, 3 * H, eq) >= 16;
  const bool k2_gemm = k1_gemm;
  if (k1_gemm) {
    eq.gen_keep = L->keep1; eq.gen_keep2 = L->keep2; eq.gen_site = 1; eq.gen_n8 = (uint64_t)T * H / 8;
    eq.gen_drop = eo.drop;
  }
  // The attention keep bits of the S <= 128 tensor-core attention are drawn
  // ahead of it by LN1 (pre-LN), whose arithmetic units idle while its row
  // loads stream, and the forward copies them in.  (Adding them to the idle
  // QKV pairs' share instead made the step 4.7 us slower at B64 S128: those
  // pairs then outlast the last round.  For longer sequences, S/8 bytes per
  // head and token, LN1 itself became compute-bound: at S = 512 it took 58
  // instead of 27 us while the attention forward saved 14 us, so there the
  // forward's helper warps draw them.)
  const bool attn_bits = aa.drop.thr && L->akeep && L->S <= 128 && attn_tc_supports(dt, aa);
  if (L->pre_ln) {
    AttnKeepGen ak = {};
    if (attn_bits) {
      ak.keep = L->akeep; ak.nh = L->nh; ak.S = L->S; ak.dp = aa.drop;
      aa.keep_ready = 1;
    }
    {
      ProfScope p_(PC_LN_FWD, s);
      ln_fwd_run(dt, x, w->ln1_g, w->ln1_b, L->h1, L->mean1, L->rstd1, T, H, L->opt.ln_eps, s,
                 keepbits && !k1_gemm ? L->keep1 : nullptr, &eo.drop, 1, &ak);
    }
    if (keepbits) eo.keep8 = L->keep1;
    gemm(L, T, 3 * H, H, L->h1, H, true, w->wqkv, H, true, eq, s);
    attn_fwd(L, aa, s);
    eo.out = L->x2;
    gemm(L, T, H, H, L->ctx, H, true, w->wo, H, true, eo, s);
    {
      ProfScope p_(PC_LN_FWD, s);
      ln_fwd_run(dt, L->x2, w->ln2_g, w->ln2_b, L->h2, L->mean2, L->rstd2, T, H, L->opt.ln_eps, s,
                 keepbits && !k2_gemm ? L->keep2 : nullptr, &e2.drop, 2);
    }
    if (keepbits) e2.keep8 = L->keep2;
    gemm(L, T, F, H, L->h2, H, true, w->w1, H, true, e1, s);
    e2.res = L->x2; e2.out = y;
    gemm(L, T, H, F, L->g, F, true, w->w2, F, true, e2, s);
  } else {
    // post-LN: the residual sums are kept unless LayerNorm backward runs from its outputs
    void* r1 = L->res1 ? L->res1 : L->dres;
    void* r2 = L->res2 ? L->res2 : L->dres;
    gemm(L, T, 3 * H, H, x, H, true, w->wqkv, H, true, eq, s);
    attn_fwd(L, aa, s);
    if (k1_gemm) eo.keep8 = L->keep1;
    eo.out = r1;
    gemm(L, T, H, H, L->ctx, H, true, w->wo, H, true, eo, s);
    {
      ProfScope p_(PC_LN_FWD, s);
      ln_fwd_run(dt, r1, w->ln1_g, w->ln1_b, L->x2, L->mean1, L->rstd1, T, H, L->opt.ln_eps, s,
                 keepbits && !k2_gemm ? L->keep2 : nullptr, &e2.drop, 2);
    }
    if (keepbits) e2.keep8 = L->keep2;
    gemm(L, T, F, H, L->x2, H, true, w->w1, H, true, e1, s);
    e2.res = L->x2; e2.out = r2;
    gemm(L, T, H, F, L->g, F, true, w->w2, F, true, e2, s);
    {
      ProfScope p_(PC_LN_FWD, s);
      ln_fwd_run(dt, r2, w->ln2_g, w->ln2_b, y, L->mean2, L->rstd2, T, H, L->opt.ln_eps, s);
    }
    if (L->yout) cudaMemcpyAsync(L->yout, y, (size_t)T * H * dtype_size(dt), cudaMemcpyDeviceToDevice, s);
  }
  st = check_cuda(L, "layer_forward");
  if (st != TL_OK) return st;
  if (L->gemm_err) {
    L->gemm_err = 0;
    return fail(L, TL_ECUDA, "a GEMM operand could not be described to the TMA unit");
  }
  L->mask = mask;
  L->have_fwd = train;
  return TL_OK;
}

tl_status layer_backward(tl_layer* L, const void* x, const void* dy, const tl_weights* w, tl_grads* g, void* dx,
                         void* stream) {
  if (!L) return TL_EINVAL;
  L->err.clear();
  if (!L->have_fwd) return fail(L, TL_ESTATE, "backward needs a preceding training-mode forward");
  if (!dy || !dx || !weights_ok(w) || !g) return fail(L, TL_EINVAL, "null tensor pointer");
  if (!g->wqkv || !g->bqkv || !g->wo || !g->bo || !g->ln1_g || !g->ln1_b || !g->w1 || !g->b1 || !g->w2 || !g->b2 ||
      !g->ln2_g || !g->ln2_b)
    return fail(L, TL_EINVAL, "null gradient pointer");
  const bool inv = L->opt.normalize_invertible != 0;
  if (!x && !(inv && L->pre_ln)) return fail(L, TL_EINVAL, "x is required (only pre-LN with normalize_invertible may omit it)");
  if (!aligned(dy) || !aligned(dx) || (x && !aligned(x))) return fail(L, TL_EINVAL, "tensor pointers must be 16-byte aligned");
  tl_status st = ensure_buffers(L);
  if (st != TL_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int dt = L->opt.dtype, T = L->T, H = L->H, F = L->F;
  const size_t es = dtype_size(dt);
  const DropoutParams dh = make_drop(L, L->ph);
  const bool keepbits = dh.thr != 0;   // the forward left the hidden-dropout keep bits
  // every parameter column sum (bias, gamma, beta gradients) leaves its
  // producer as partial rows in a slot of its own; one launch at the end sums
  // them.  Stochastic mode: the producers add them into the gradients
  // themselves (zeroed first) with atomics, and so do the splits of a
  // split-K weight gradient; nothing is left for a closing launch.
  const bool relaxed = L->opt.stochastic_mode != 0;
  FinalizeList fin;
  fin.n = 0;
  auto slot = [&](int i) { return L->part + (size_t)i * L->part_floats; };
  // where column sum `i` of gradient `out` goes
  auto sink = [&](int i, float* out) { return relaxed ? out : slot(i); };
  auto finish = [&](const FinalizeJob& j) {
    if (!relaxed) fin.job[fin.n++] = j;
  };
  if (relaxed) {
    ZeroList z;
    z.count = 0;
    auto zero = [&](float* p, size_t n) {
      z.p[z.count] = p;
      z.n[z.count++] = n;
    };
    zero(g->bqkv, 3 * (size_t)H); zero(g->bo, H); zero(g->ln1_g, H); zero(g->ln1_b, H);
    zero(g->b1, F); zero(g->b2, H); zero(g->ln2_g, H); zero(g->ln2_b, H);
    // the weight gradients whose K is split (those with split-K scratch)
    if (L->splitk[0]) zero(g->w2, (size_t)H * F);
    if (L->splitk[1]) zero(g->w1, (size_t)F * H);
    if (L->splitk[2]) zero(g->wo, (size_t)H * H);
    if (L->splitk[3]) zero(g->wqkv, (size_t)3 * H * H);
    ProfScope p_(PC_ROWWISE, s);
    zero_list_run(z, s);
  }

  auto ln_bwd = [&](const void* dyln, const void* xin, const void* yln, const float* mean, const float* rstd,
                    const void* gamma, const void* beta, const void* res, void* dxo, void* drop_out, int site,
                    float* dgamma, float* dbeta, float* dsum, int slot0, const uint8_t* keep8) {
    LnBwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.dy = dyln; a.x = inv ? nullptr : xin; a.y = inv ? yln : nullptr;
    a.mean = mean; a.rstd = rstd; a.gamma = gamma; a.beta = beta;
    a.res = res; a.dx = dxo; a.drop_out = drop_out; a.drop = dh; a.site = site; a.keep8 = keep8;
    a.part_dgamma = sink(slot0, dgamma); a.part_dbeta = sink(slot0 + 1, dbeta);
    a.part_dsum = drop_out ? sink(slot0 + 2, dsum) : nullptr;
    a.part_acc = relaxed ? 1 : 0;
    a.rows = T; a.H = H;
    ProfScope p_(PC_LN_BWD, s);
    const int parts = ln_bwd_run(dt, a, s);
    finish({a.part_dgamma, dgamma, parts, H, 0});
    finish({a.part_dbeta, dbeta, parts, H, 0});
    if (drop_out) finish({a.part_dsum, dsum, parts, H, 0});
  };

  // FFN block: dZ2 -> dW2, dU (into big), db1, then dW1 with the FFN input
  // gradient dU W1 (epilogue `edin`, output (T, H))
  auto ffn_bwd = [&](const void* ffn_in, const EpiParams& edin, int db1_slot) {
    EpiParams ew2 = epi(EPI_F32, g->w2, F);
    ew2.accumulate = relaxed;
    if (L->opt.gelu_checkpoint) {
      ProfScope p_(PC_ROWWISE, s);
      gelu_run(dt, L->u, L->big, (size_t)T * F, L->opt.gelu_tanh ? 1 : 0, s);
    }
    // dU = (dZ2 W2) * GELU'(U): GELU' from U (checkpoint mode) or as stored by the forward
    EpiParams edu = epi(L->opt.gelu_checkpoint ? EPI_DGELU : EPI_MUL, L->big, F);
    edu.aux = L->u;
    edu.gelu_tanh = L->opt.gelu_tanh ? 1 : 0;
    // the tensor-core GEMM sums dU's columns in its epilogue (db1)
    const bool fused_db1 = gemm_uses_tensor_cores(dt) != 0;
    if (fused_db1) edu.colsum = sink(db1_slot, g->b1);
    edu.accumulate = relaxed;
    GemmDesc gw2 = wdesc(L, 0, &fin, H, F, T, L->dz2, H, L->g, F);                // dW2 = dZ2^T G
    // recompute mode: G was just rewritten by the GELU launch before this one
    if (L->opt.gelu_checkpoint) gw2.b_early = false;
    const GemmDesc gdu = gdesc(L, T, F, H, L->dz2, H, true, w->w2, F, false);   // dU = (dZ2 W2) GELU'(U)
    if (L->g != L->big) {
      gemm2(L, gw2, ew2, gdu, edu, s);
    } else {
      // recompute mode: G lives where dU goes, so dW2 must finish first
      ProfScope p_(PC_GEMM, s);
      if (gemm_run(dt, gw2, ew2, s) != 0 || gemm_run(dt, gdu, edu, s) != 0) L->gemm_err = 1;
    }
    if (fused_db1) finish({slot(db1_slot), g->b1, (T + 255) / 256 * 8, F, 0});   // db1 from the GEMM
    else bias_grad(L, L->big, F, db1_slot, g->b1, fin, s);                                  // db1
    EpiParams ew1 = epi(EPI_F32, g->w1, H);
    ew1.accumulate = relaxed;
    gemm2(L, wdesc(L, 1, &fin, F, H, T, L->big, F, ffn_in, H), ew1,          // dW1 = dU^T in
          gdesc(L, T, H, F, L->big, F, true, w->w1, H, false), edin, s);   // dU W1
  };
  // attention block from dA: dWo with dctx, attention backward, dbqkv, then
  // dWqkv with the attention input gradient dQKV Wqkv (epilogue `edin`)
  auto attn_bwd_block = [&](const void* attn_in, const EpiParams& edin, int dbqkv_slot) {
    EpiParams ewo = epi(EPI_F32, g->wo, H);
    ewo.accumulate = relaxed;
    EpiParams edc = epi(EPI_STORE, L->dctx, H);
    gemm2(L, wdesc(L, 2, &fin, H, H, T, L->da, H, L->ctx, H), ewo,           // dWo = dA^T ctx
          gdesc(L, T, H, H, L->da, H, true, w->wo, H, false), edc, s);     // dctx = dA Wo
    AttnArgs aa = attn_args(L, L->mask);
    const bool fused_dbqkv = attn_tc_supports(dt, aa) && attn_tc_fuses_colsum(dt, aa);
    if (fused_dbqkv) {
      aa.colsum = sink(dbqkv_slot, g->bqkv);
      aa.colsum_acc = relaxed ? 1 : 0;
    }
    attn_bwd(L, aa, s);
    if (fused_dbqkv) finish({slot(dbqkv_slot), g->bqkv, L->B * 4, 3 * H, 0});   // from the attention
    else bias_grad(L, L->dqkv, 3 * H, dbqkv_slot, g->bqkv, fin, s);
    EpiParams ewq = epi(EPI_F32, g->wqkv, H);
    ewq.accumulate = relaxed;
    gemm2(L, wdesc(L, 3, &fin, 3 * H, H, T, L->dqkv, 3 * H, attn_in, H), ewq,           // dWqkv = dQKV^T in
          gdesc(L, T, H, 3 * H, L->dqkv, 3 * H, true, w->wqkv, H, false), edin, s);  // dQKV Wqkv
  };

  if (L->pre_ln) {
    {
      ProfScope p_(PC_ROWWISE, s);
      dropout_rows_run(dt, dy, L->dz2, dh, 2, T, H, sink(0, g->b2), s, keepbits ? L->keep2 : nullptr, relaxed);
      finish({slot(0), g->b2, rowdrop_parts(T), H, 0});
    }
    ffn_bwd(L->h2, epi(EPI_STORE, L->dh, H), 1);                         // dH2 = dU W1
    ln_bwd(L->dh, L->x2, L->h2, L->mean2, L->rstd2, w->ln2_g, w->ln2_b, dy, L->dx2, L->da, 1,
           g->ln2_g, g->ln2_b, g->bo, 2, keepbits ? L->keep1 : nullptr);
    attn_bwd_block(L->h1, epi(EPI_STORE, L->dh, H), 5);                  // dH1 = dQKV Wqkv
    ln_bwd(L->dh, x, L->h1, L->mean1, L->rstd1, w->ln1_g, w->ln1_b, L->dx2, dx, nullptr, 0,
           g->ln1_g, g->ln1_b, nullptr, 6, nullptr);
  } else {
    const void* r2 = L->res2;
    const void* r1 = L->res1;
    ln_bwd(dy, r2, L->yout, L->mean2, L->rstd2, w->ln2_g, w->ln2_b, nullptr, L->dres, L->dz2, 2,
           g->ln2_g, g->ln2_b, g->b2, 0, keepbits ? L->keep2 : nullptr);
    EpiParams edx2 = epi(EPI_STORE, L->dx2, H);
    edx2.res = L->dres;
    ffn_bwd(L->x2, edx2, 3);                                              // dx2 = dU W1 + dres2
    ln_bwd(L->dx2, r1, L->x2, L->mean1, L->rstd1, w->ln1_g, w->ln1_b, nullptr, L->dres, L->da, 1,
           g->ln1_g, g->ln1_b, g->bo, 4, nullptr);
    EpiParams edx = epi(EPI_STORE, dx, H);
    edx.res = L->dres;
    attn_bwd_block(x, edx, 7);                                            // dx = dQKV Wqkv + dres1
  }
  {
    ProfScope p_(PC_ROWWISE, s);
    colsum_finalize_list_run(fin, s);                                     // every bias / LayerNorm gradient
  }
  (void)es;
  st = check_cuda(L, "layer_backward");
  if (st == TL_OK && L->gemm_err) {
    L->gemm_err = 0;
    return fail(L, TL_ECUDA, "a GEMM operand could not be described to the TMA unit");
  }
  return st;
}

tl_status tl_device_check(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return TL_ECUDA;
  return device_take_error() ? TL_ETIMEOUT : TL_OK;
}

tl_status tl_set_wait_limit_ns(uint64_t ns) {
  device_set_wait_limit(ns);
  return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ECUDA;
}

tl_status tl_wait_probe(void* stream) {
  gemm_tc_wait_probe((cudaStream_t)stream);
  return cudaPeekAtLastError() == cudaSuccess ? TL_OK : TL_ECUDA;
}

tl_status tl_gelu_eval(const float* u, float* g, float* dg, uint64_t n, void* stream) {
  if (!u || !g || !dg) return TL_EINVAL;
  if (n == 0) return TL_OK;
  gelu_eval_run(u, g, dg, n, 0, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ECUDA;
}

tl_status tl_gelu_tanh_eval(const float* u, float* g, float* dg, uint64_t n, void* stream) {
  if (!u || !g || !dg) return TL_EINVAL;
  if (n == 0) return TL_OK;
  gelu_eval_run(u, g, dg, n, 1, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ECUDA;
}

tl_status tl_dropout_keep_mask(uint64_t seed, uint64_t philox_offset, int site, float p, uint64_t e0, uint64_t n,
                               uint8_t* keep, void* stream) {
  if (!keep || (e0 % 8) || (n % 8) || !(p >= 0.0f && p < 1.0f) || site < 0) return TL_EINVAL;
  if (n == 0) return TL_OK;
  DropoutParams d;
  d.seed = seed;
  d.offset = philox_offset;
  d.thr = (uint32_t)std::floor((double)p * 65536.0);
  d.scale = 1.0f / (1.0f - p);
  dropout_mask_run(d, site, e0, n, keep, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ECUDA;
}

}  // extern "C"
