// Internal declarations shared by the C-ABI layer (vt_api.cpp) and the kernel
// translation units.  Not part of the public interface (include/vt.h is).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "vt.h"

namespace vt {

// Token order of the activations of one image.
enum TokenOrder : int { ORDER_RASTER = 0, ORDER_BLOCK = 1 };

// Maximum position along any grid axis that the RoPE tables cover.
constexpr int kRopeMaxPos = 4096;
// Pairs per axis the tables hold (head_dim up to 2 * 3 * 32).
constexpr int kRopePairs = 32;

// Decodes token n of an image with grid (gt, gh, gw) in the given order into its
// (t, h, w) patch position.  Block order lists the 4 members of every 2x2 group
// consecutively: (0,0), (0,1), (1,0), (1,1); groups follow raster order.
__host__ __device__ inline void token_position(int n, int gh, int gw, int order, int* t, int* h, int* w) {
  const int per_t = gh * gw;
  *t = n / per_t;
  const int r = n - *t * per_t;
  if (order == ORDER_BLOCK) {
    const int m = r >> 2, q = r & 3, hw2 = gw >> 1;
    const int i = m / hw2, j = m - (m / hw2) * hw2;
    *h = 2 * i + (q >> 1);
    *w = 2 * j + (q & 1);
  } else {
    *h = r / gw;
    *w = r - (r / gw) * gw;
  }
}

// --------------------------------------------------- variable-resolution batches

// Images of different grids packed into one token sequence.  Passed by value as a
// kernel parameter (so launches stay capturable in CUDA graphs).
constexpr int kMaxVarlenImages = 64;
struct VarlenTable {
  int count;                              // images in the batch
  int tok_off[kMaxVarlenImages + 1];      // first token of each image; tok_off[count] = total
  int gh[kMaxVarlenImages];               // patch grid of each image (t = 1)
  int gw[kMaxVarlenImages];
  long long vt_off[kMaxVarlenImages];     // element offset of each image's v^T block
  int ld_vt[kMaxVarlenImages];            // its row stride (tokens rounded up to 8)
  long long pix_off[kMaxVarlenImages];    // float offset of each image's [3, H, W] pixels
};

// Image of packed token `row` (binary search over tok_off).
__host__ __device__ inline int varlen_image(const VarlenTable& t, int row) {
  int lo = 0, hi = t.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t.tok_off[mid] <= row) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ GEMM

// ACT_DGELU_*: backward of GELU, out = (A W^T) * gelu'(aux) with aux passed as `resid`
// (the pre-activation; not added).
enum GemmAct : int { ACT_NONE = 0, ACT_GELU_TANH = 1, ACT_GELU_ERF = 2, ACT_DGELU_TANH = 3, ACT_DGELU_ERF = 4 };

// out[M, N] = act(A[M, K] * W[N, K]^T + bias) (+ resid), bf16 in and out, fp32 accumulate.
struct GemmParams {
  int M, N, K;
  const void* A;      // [M, lda] bf16
  int lda;            // elements, multiple of 8
  const void* W;      // [N, ldw] bf16
  int ldw;
  const void* bias;   // [N] bf16 or null
  const void* resid;  // [M, ldr] bf16 or null (may alias out)
  int ldr;
  void* out;          // [M, ldo] bf16
  int ldo;
  int act;
  void* pre_out;  // optional [M, ldo] bf16: the values before the activation (bias added)
  // QKV mode: output columns are [q | k | v], each heads*head_dim wide.  q and k are
  // rotated (3D RoPE) and written [B, heads, ntok, head_dim]; v is written transposed
  // [B, heads, head_dim, ld_vt].
  void* q;
  void* k;
  void* vt;
  int heads, head_dim, ntok, ld_vt;
  int gt, gh, gw, order;
  int rope;                 // 0: no rotation
  int sections[3];
  const float2* rope_tab;   // [3][kRopeMaxPos][kRopePairs] (cos, sin)
  // Variable-resolution batch: rows are packed tokens of images of different grids.
  // q and k of image b are [heads, N_b, head_dim] blocks starting at token tok_off[b];
  // v^T of image b is [heads, head_dim, ld_vt[b]] at vt_off[b].
  int varlen;
  VarlenTable vl;
  // Split-K tail of plain products on CTA pairs (sk_part null: off).  The caller gives
  // sk_part, gemm_split_bytes() bytes of fp32 scratch; launch_gemm sets the rest when
  // the output tiles leave the last round of the grid mostly idle: the first sk_full
  // tiles run whole, each remaining tile's K steps are cut into sk_split ranges, one per
  // idle CTA pair, and a second kernel adds their fp32 partial sums in a fixed order and
  // applies the epilogue.
  float* sk_part;
  int sk_full, sk_split;
  // Tile order (set by launch_gemm): 0 walks the row tiles of A fastest, so that the CTAs
  // running together share each tile of W through L2; 1 walks the column tiles fastest,
  // so that they share each row tile of A (used when A is the larger operand, which is
  // then read from memory once).
  int n_fastest;
};

// Bytes of split-K scratch a product may use (one 256 x 256 fp32 tile per CTA pair).
size_t gemm_split_bytes();

// Returns a CUDA error code (cudaSuccess on success); host-side shape checks are the
// caller's job.
// *kernels (if given) receives the number of kernels launched (2 with a split-K tail sum).
cudaError_t launch_gemm(const GemmParams& p, cudaStream_t stream, int qkv_mode, int* kernels = nullptr);
unsigned int gemm_read_clear_error(cudaStream_t stream);

// ------------------------------------------------------------- attention

struct AttnParams {
  const void* q;   // [B, H, N, D] bf16, rotated
  const void* k;   // [B, H, N, D] bf16, rotated
  const void* vt;  // [B, H, D, ld_vt] bf16
  void* o;         // [B, N, H * D] bf16
  int B, H, N, D, ld_vt;
  float scale;
  // Variable-resolution batch (varlen != 0): image b has vl.tok_off[b+1] - tok_off[b]
  // tokens; q and k hold [H, N_b, D] blocks at token tok_off[b]; vt is [B, H, D, ld_vt]
  // with one common ld_vt >= every N_b and zeros beyond N_b; o rows are packed tokens.
  // N is then the largest N_b (it sizes the grid).
  int varlen;
  VarlenTable vl;
  // Optional: base-2 log-sum-exp of the scaled scores of every query row,
  // lse[(b*H + h) * ld_lse + n] = log2(sum_j 2^(s_nj * scale * log2 e)), for the backward.
  float* lse;
  int ld_lse;
  // Work schedule (set by launch_attention; callers leave it zero): the first sched_full
  // items run whole in rounds of the grid, then sched_tail_pairs items form a tail of one
  // unit per CTA, sched_tail_split of them cut into two single-tile units.
  int sched_full, sched_tail_pairs, sched_tail_split;
};
cudaError_t launch_attention(const AttnParams& p, cudaStream_t stream);
unsigned int attention_read_clear_error(cudaStream_t stream);

// Attention backward for uniform batches (every image N tokens).  q, k, v, o-gradient
// and the forward's lse in; dq, dk (rotated back by RoPE) and dv written into the
// [B*N, ld_dqkv] qkv-gradient matrix at column blocks 0, H*D and 2*H*D.
struct AttnBwdParams {
  const void* q;      // [B, H, N, D] bf16, rotated
  const void* k;      // [B, H, N, D] bf16, rotated
  const void* vt;     // [B, H, D, ld] bf16 (v transposed, as the forward uses it)
  const void* dO;     // [B*N, H*D] bf16, gradient of the attention output
  const float* lse;   // [B*H, ld_stats], from the forward
  const float* delta; // [B*H, ld_stats], rowsum(dO * O) per query
  int ld_stats;       // multiple of 64, >= N
  void* dqkv;         // [B*N, ld_dqkv] bf16
  int ld_dqkv;
  int B, H, N, D, ld;  // ld: multiple of 8, >= N
  float scale;
  int rope;
  int sections[3];
  const float2* rope_tab;
  int gh, gw, order;
};
cudaError_t launch_attention_backward(const AttnBwdParams& p, cudaStream_t stream);
unsigned int attention_bwd_read_clear_error(cudaStream_t stream);

// -------------------------------------------------------- memory-bound ops

cudaError_t launch_layernorm(const void* x, const void* gamma, const void* beta, void* y, int rows, int cols,
                             float eps, cudaStream_t stream);
// pixels [B, 3, H, W] fp32 -> patch vectors [B * gh * gw, 3 * tp * p * p] bf16 in `order`.
cudaError_t launch_patch_unfold(const float* pixels, void* out, int B, int H, int W, int patch, int tp,
                                int order, cudaStream_t stream);
// Clips [B, F, 3, H, W] -> [B * ceil(F/tp) * gh * gw, 3 * tp * p * p]; temporal patch t
// takes frames t*tp .. t*tp+tp-1, the last frame repeated past the end of the clip.
cudaError_t launch_patch_unfold_frames(const float* pixels, void* out, int B, int F, int H, int W, int patch,
                                       int tp, int order, cudaStream_t stream);
// Packed images of different sizes (vl.pix_off, vl.gh, vl.gw) -> packed patch vectors
// in 2x2-block order per image.
cudaError_t launch_patch_unfold_varlen(const float* pixels, void* out, const VarlenTable& vl, int patch, int tp,
                                       cudaStream_t stream);
// Decoded 8-bit RGB images [H0_b, W0_b, 3] resized to one patch grid.  Passed by value.
constexpr int kMaxShrink = 16;  // a source side may be at most 16x the target side
struct PreprocTable {
  int count;                            // images in this launch (<= kMaxVarlenImages)
  long long src_off[kMaxVarlenImages];  // byte offset of each image
  int src_h[kMaxVarlenImages];
  int src_w[kMaxVarlenImages];
  float mean[3], std[3];                // per channel, applied after scaling by 1/255
};
// Upper bound on the source rows under one output patch (sizes the shared staging).
size_t preprocess_rows_bound(int src, int dst, int patch);
// Bicubic resize + normalisation of tab.count images to grid (gh, gw): to_patches = 0
// writes pixels fp32 [count, 3, gh*p, gw*p]; to_patches = 1 writes patch vectors bf16
// [count*gh*gw, 3*tp*p*p] in `order`.  rows_cap >= preprocess_rows_bound of every image.
cudaError_t launch_preprocess(const uint8_t* images, const PreprocTable& tab, void* out, int gh, int gw,
                              int patch, int tp, int order, int to_patches, int rows_cap, cudaStream_t stream);
unsigned int preprocess_read_clear_error(cudaStream_t stream);
// Row gather: out[r] = in[src(r)] where src maps between raster and block order.
// to_block != 0: out is block order, in is raster.  Rows of `cols` bf16 each.
cudaError_t launch_reorder_rows(const void* in, void* out, int B, int gt, int gh, int gw, int cols, int to_block,
                                cudaStream_t stream);
// q, k [B, H, N, D] -> rotated copies; v [B, H, N, D] -> vt [B, H, D, ld_vt].
// pos: device [N, 3] int32 (t, h, w) or null for no rotation.
cudaError_t launch_attention_prep(const void* q, const void* k, const void* v, void* qr, void* kr, void* vt,
                                  int B, int H, int N, int D, int ld_vt, const int32_t* pos,
                                  const int sections[3], float theta, cudaStream_t stream);

// ---------------------------------------------------------- backward, memory-bound

// dx = dres + LayerNorm backward of x (gamma) applied to dy; dres may alias dx.
cudaError_t launch_layernorm_backward(const void* x, const void* gamma, const void* dy, const void* dres, void* dx,
                                      int rows, int cols, float eps, cudaStream_t stream);
// delta[(b*H + h) * ld + n] = <dO, O> over head h of token b*N + n ([B*N, H*D] bf16 each).
cudaError_t launch_attention_delta(const void* dO, const void* O, float* delta, int B, int N, int H, int D, int ld,
                                   cudaStream_t stream);
// For z = (b, h): out[c][r] = in[r][c], r < R, c < C; strides in bf16 elements.
cudaError_t launch_transpose(const void* src, void* dst, int B, int H, int R, int C, long in_sb, long in_sh,
                             long in_ld, long out_sb, long out_sh, long out_ld, cudaStream_t stream);
// Patch-vector gradients [B*gh*gw, 3*tp*p*p] (tokens in `order`) -> pixel gradients
// [B, 3, H, W] fp32 (sum over the repeated frames).
cudaError_t launch_patch_fold(const void* du, float* dpixels, int B, int H, int W, int patch, int tp, int order,
                              cudaStream_t stream);

// -------------------------------------------------------------------- TMA

// Creates a 2D tiled tensor map over a row-major bf16 matrix [rows, cols] with row
// stride ld (elements) and box [box_rows, box_cols]; swizzle_bytes in {0, 32, 64, 128}.
bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                  uint32_t box_rows, uint32_t box_cols, int swizzle_bytes);

int device_sm_count();

unsigned int selftest_read_clear_error(cudaStream_t stream);

// Sets the calling thread's message returned by vt_last_error().
void set_error_message(const char* msg);

// Host side of the stand-alone attention, shared by the entry points that take a
// workspace and the one with static scratch: argument checks (positive sizes and
// scale, a head_dim with a kernel, B * H * N rows within the 32-bit index range), and
// the two launches, each bracketed for the launch trace and the profiler.
vt_status check_attention_dims(int B, int H, int N, int D, float scale);
vt_status run_attention_prep(const void* q, const void* k, const void* v, void* qr, void* kr, void* vt_, int B, int H,
                             int N, int D, int ld_vt, const int32_t* pos, const int sections[3], float theta,
                             cudaStream_t st);
vt_status run_attention(const AttnParams& p, cudaStream_t st);

}  // namespace vt
