// kernels.h — host-side launchers of the layer's kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace tlp {

enum Dtype { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };

// Launches `kernel` with programmatic stream serialization (see pdl_wait in
// common.cuh); the kernel must call pdl_wait() before touching global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}
inline size_t dtype_size(int dt) { return dt == DT_F32 ? 4 : 2; }

// ------------------------------------------------------------------ GEMM
// C[m, n] = sum_k A(m, k) * B(n, k), float32 accumulation, then an epilogue.
// A(m, k) = A[m*lda + k] when a_kmajor, else A[k*lda + m]; B likewise.
struct FinalizeList;

struct GemmDesc {
  int M, N, K;
  const void* A; int lda; bool a_kmajor;
  const void* B; int ldb; bool b_kmajor;
  float* splitk_ws;          // float32 scratch for split-K weight gradients, or null
  size_t splitk_ws_floats;
  // when set (and it has room), a split-K float32 GEMM appends the sum of its
  // partials to this list (summed by a later colsum_finalize_list_run; the
  // scratch must stay untouched until then) instead of launching the sum
  FinalizeList* defer = nullptr;
  // B was not written by the kernel launched just before this GEMM on its
  // stream (a weight, or an activation of an earlier kernel): the tensor-core
  // kernel then loads its first stages of B before it waits for that kernel
  bool b_early = false;
};

enum EpiKind {
  EPI_QKV = 0,        // + bias, scattered into Q, K, V laid out (B, heads, S, d)
  EPI_BIAS_DROP_RES,  // out = res + dropout(acc + bias); element index m*N + n
  EPI_BIAS_GELU,      // U = acc + bias (stored), G = GELU(stored U) (stored if out2)
  EPI_DGELU,          // out = acc * GELU'(U) (GELU'(U) rounded to storage first)
  EPI_STORE,          // out = acc (+ res if given)
  EPI_F32,            // float32 out = acc
  EPI_BIAS_GELU_D,    // U = acc + bias rounded to storage; out = GELU'(U), out2 = G = GELU(U)
  EPI_MUL             // out = acc * aux (aux = the GELU'(U) that EPI_BIAS_GELU_D stored)
};

struct EpiParams {
  int kind;
  const void* bias;   // N entries, storage type
  const void* res;    // residual (M, N) storage type, or null
  const void* aux;    // EPI_DGELU: U (M, N); EPI_MUL: the factor (M, N)
  void* out;          // (M, N) with row stride ldo (EPI_QKV: Q|K|V base)
  void* out2;         // EPI_BIAS_GELU: G, may be null; EPI_BIAS_GELU_D: G
  int ldo;
  // dropout (EPI_BIAS_DROP_RES)
  DropoutParams drop;
  int site;
  const uint8_t* keep8;   // EPI_BIAS_DROP_RES: precomputed keep bits (byte per 8 elements), or null
  // head split (EPI_QKV)
  int seq, hidden, head_dim, heads, tokens;
  // EPI_BIAS_GELU / EPI_BIAS_GELU_D / EPI_DGELU: 1 for the tanh approximation of GELU
  int gelu_tanh;
  // EPI_QKV / EPI_BIAS_DROP_RES on the tensor-core pair kernel: the CTA
  // pairs left without a tile in the last round (gemm_tc_bubble_pairs) draw
  // the keep bits of dropout site gen_site with gen_drop (gen_n8 bytes, one
  // per 8 elements) into gen_keep meanwhile, and those of site gen_site + 1
  // into gen_keep2 when it is set; or null
  uint8_t* gen_keep;
  uint8_t* gen_keep2;
  int gen_site;
  uint64_t gen_n8;
  DropoutParams gen_drop;
  // EPI_DGELU / EPI_MUL on the tensor-core GEMM: column sums of the stored output, one
  // partial row per (256-row tile, CTA of the pair, TMEM lane quarter), i.e.
  // row (m / 256) * 8 + ((m % 256) / 128) * 4 + (m % 128) / 32; or null
  float* colsum;
  // 1: add instead of store (arrival order, not a fixed one).  EPI_F32 on the
  // tensor-core GEMM: the split-K partial tiles are added into `out` (by TMA
  // reduce-add; no workspace, no closing sum), so `out` must hold zeros when
  // K is split; `colsum`: every partial row is added into its single row
  // (cols floats, which must hold zeros)
  int accumulate;
};

// CTA pairs of the tensor-core pair kernel that have no tile in its last
// round for an M x N GEMM with this epilogue (0 when it runs elsewhere or the
// last round is full): the pairs that honour EpiParams.gen_keep.
int gemm_tc_bubble_pairs(int dtype, int M, int N, const EpiParams& e);

// Returns 0, or non-zero when an operand cannot be described to the TMA unit
// (unaligned base address or row stride).
int gemm_run(int dtype, const GemmDesc& g, const EpiParams& e, cudaStream_t s);
// Two independent GEMMs (a float32 weight gradient `ga` and an input
// gradient `gb` that reads the same operands), in one launch where the
// tensor-core kernel can plan them together; same results as two gemm_run.
int gemm_run2(int dtype, const GemmDesc& ga, const EpiParams& ea, const GemmDesc& gb, const EpiParams& eb,
              cudaStream_t s);
// 1 when the tensor-core (tcgen05) GEMM serves this dtype, 0 for the SIMT one.
int gemm_uses_tensor_cores(int dtype);
// Split-K scratch (floats) the tensor-core GEMM would use for an EPI_F32 GEMM of this shape.
size_t gemm_splitk_ws_floats(int dtype, int M, int N, int K);
// Reads and clears the error word set by a bounded device-side wait that gave up.
int device_take_error();
// Sets the limit (ns; 0 = the default 2 s) of every kernel's bounded waits on
// the current device.  Synchronous.
void device_set_wait_limit(uint64_t ns);
// Launches a kernel whose one bounded wait nothing ever satisfies (it gives
// up after the limit and sets the error word of the GEMM kernels).
void gemm_tc_wait_probe(cudaStream_t s);

// ------------------------------------------------------------------ LayerNorm
// LayerNorm forward.  With keep_out, also writes the dropout keep bits of
// site `site` for the (rows, H) elements: byte e/8 holds elements e..e+7
// (bit k = element e+k), the same bits dropout_bits8 gives; the row kernels
// have idle arithmetic units, so the downstream kernels read the bits
// instead of drawing Philox themselves.
// With AttnKeepGen.keep set, a pre-LN LayerNorm forward (whose rows are the
// layer's tokens, row t = b*S + s) also draws the attention-probability keep
// bits (site 0) whose query row is its token, for every head, in the S <= 128
// layout of AttnArgs.keep (byte q of query s of item (b, h), at
// ((b*nh + h)*128 + s)*16 + q, is element group (((b*nh + h)*S + s)*S)/8 + q),
// so the attention forward reads them.
struct AttnKeepGen {
  uint8_t* keep;       // null: off
  int nh, S;
  DropoutParams dp;
};
void ln_fwd_run(int dtype, const void* x, const void* gamma, const void* beta, void* y, float* mean,
                float* rstd, int rows, int H, float eps, cudaStream_t s, uint8_t* keep_out = nullptr,
                const DropoutParams* dp = nullptr, int site = 0, const AttnKeepGen* akeep = nullptr);

// LayerNorm backward of one row block + residual-gradient add + optional
// dropout of the result, with column partial sums for dgamma, dbeta and the
// sum of the dropped output.  Partials are (nparts, H) float32 each.
struct LnBwdArgs {
  const void* dy;       // gradient w.r.t. the LayerNorm output (rows, H)
  const void* x;        // LayerNorm input (rows, H), or null when invertible
  const void* y;        // LayerNorm output (invertible mode), else null
  const float* mean;
  const float* rstd;
  const void* gamma;
  const void* beta;     // invertible mode
  const void* res;      // added to dx, or null
  void* dx;             // (rows, H)
  void* drop_out;       // dropout(dx) (rows, H), or null
  DropoutParams drop;
  int site;
  const uint8_t* keep8;   // keep bits of the dropout copy (byte per 8 elements), or null: draw them
  float* part_dgamma;
  float* part_dbeta;
  float* part_dsum;     // column sums of drop_out, or null
  int rows, H;
  // 1: every block adds its column sums into row 0 of part_* (the gradients
  // themselves, holding zeros) with atomics instead of storing its own row
  int part_acc;
};
// Upper bound of the partial rows ln_bwd_run writes (size of the part_* buffers).
int ln_bwd_parts(int rows);
// Returns the number of partial rows written (to pass to the finalize).
int ln_bwd_run(int dtype, const LnBwdArgs& a, cudaStream_t s);

// ------------------------------------------------------------------ elementwise / reductions
// out = dropout(in) (site, element t*H + c) with column partial sums of out.
int rowdrop_parts(int rows);
// With acc, every block adds its column sums into part_sum[0..H) (holding
// zeros) with atomics instead of storing a row of its own.
void dropout_rows_run(int dtype, const void* in, void* out, const DropoutParams& dp, int site, int rows, int H,
                      float* part_sum, cudaStream_t s, const uint8_t* keep8 = nullptr, int acc = 0);
// Column partial sums of a (rows, cols) storage-typed matrix: (colsum_parts(rows), cols) floats
// (with acc: added into part[0..cols), holding zeros, with atomics).
int colsum_parts(int rows);
void colsum_run(int dtype, const void* X, int rows, int cols, float* part, cudaStream_t s, int acc = 0);
// Sets every listed float32 buffer to zero, in one launch.
constexpr int kMaxZero = 16;
struct ZeroList {
  float* p[kMaxZero];
  size_t n[kMaxZero];
  int count;
};
void zero_list_run(const ZeroList& z, cudaStream_t s);
// out[c] = sum_p part[p*cols + c] (fixed order).
void colsum_finalize_run(const float* part, int nparts, int cols, float* out, cudaStream_t s);
// Several finalizes in one launch, each job either
//   stride == 0: out[c] = sum over p < nparts of part[p * cols + c] (column
//                sums of partial rows), or
//   stride != 0: out[i] = sum over p < nparts of part[p * stride + i] for
//                i < cols (the split-K partials of a float32 weight gradient;
//                cols a multiple of 4, 16-byte aligned pointers),
// always summed in increasing p.
constexpr int kMaxFinalize = 8;        // partial-row slots a layer keeps
constexpr int kMaxFinalizeJobs = 12;   // + the split-K weight gradients
struct FinalizeJob {
  const float* part;
  float* out;
  int nparts, cols;
  size_t stride;
};
struct FinalizeList {
  FinalizeJob job[kMaxFinalizeJobs];
  int n;
};
void colsum_finalize_list_run(const FinalizeList& fl, cudaStream_t s);
// The same for up to three (partials, output) pairs in one launch (p1/p2 may be null).
void colsum_finalize3_run(const float* p0, const float* p1, const float* p2, float* o0, float* o1, float* o2,
                          int nparts, int cols, cudaStream_t s);
// g[i] = GELU(u[i]), dg[i] = GELU'(u[i]) with the device GELU every kernel uses (float32).
void gelu_eval_run(const float* u, float* g, float* dg, uint64_t n, int tanh_form, cudaStream_t s);
// G = GELU(U), elementwise, n a multiple of 8.
void gelu_run(int dtype, const void* U, void* G, size_t n, int tanh_form, cudaStream_t s);
// keep[i] = dropout keep bit of element e0 + i of `site`.
void dropout_mask_run(const DropoutParams& dp, int site, uint64_t e0, uint64_t n, uint8_t* keep, cudaStream_t s);

// ------------------------------------------------------------------ attention
struct AttnArgs {
  int B, S, nh, d;
  const void* q;        // (B, nh, S, d)
  const void* k;
  const void* v;
  const float* mask;    // (B, S) additive or null
  float scale;          // 1/sqrt(d)
  DropoutParams drop;   // site 0
  void* ctx;            // (B*S, nh*d)
  float* lse;           // (B, nh, S); +inf marks a row with every key masked
  // attention dropout keep bits of the tensor-core path (bit k of byte c =
  // key 8c + k of a query row): the forward writes them, the backward reads
  // them instead of drawing Philox again; null to draw them in both.  Laid
  // out [B*nh][128 query rows][16 bytes] for S <= 128, else [B*nh][S][S/8]
  // (byte e/8 for the flat element index e of site 0)
  uint8_t* keep;
  // 1: the S <= 128 keep bits are already in `keep` (drawn by the LayerNorm
  // forward before the attention), the forward reads them instead of drawing
  int keep_ready;
  // (B) ints the forward of sequences longer than 128 fills with one past
  // each sequence's last unmasked key (key tiles beyond it are skipped), or
  // null to run every key tile
  int* kv_ext;
  // backward
  const void* dctx;     // (B*S, nh*d)
  float* dvec;          // (B, nh, S) rowsum(dctx * ctx)
  void* dqkv;           // (B*S, 3*nh*d): [dQ | dK | dV]
  // column sums of the stored dQKV (the QKV bias gradient), one partial row
  // per (sequence b, 32-query block q): row b*4 + q of a (B*4, 3*nh*d)
  // float32 matrix; written only by kernels that fuse it (see
  // attn_tc_fuses_colsum), else untouched
  float* colsum;
  // 1: the partial rows are added into row 0 of `colsum` (holding zeros)
  // with atomics instead
  int colsum_acc;
};
void attn_fwd_run(int dtype, const AttnArgs& a, cudaStream_t s);
void attn_bwd_run(int dtype, const AttnArgs& a, cudaStream_t s);

}  // namespace tlp
