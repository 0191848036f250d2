// Image preprocessing on the GPU: decoded 8-bit RGB images [H0, W0, 3] of any size are
// resized (bicubic), scaled by 1/255 and normalised per channel, and written either as
// model pixels [3, H, W] fp32 or straight into the patch-embedding GEMM's A operand
// (patch vectors in (c, t, kh, kw) order, the frame repeated over the temporal patch).
//
// Source: "v2_loaders - Differentiable Vision Tower Loaders (spark2)", section 3
// (MiniMax-M3 vision tower): bicubic resize, OpenAI CLIP mean/std, patchify with the
// temporal dimension padded to 2 by repeating the frame.  The resize is cubic
// convolution with Keys' kernel at a = -0.5: output pixel centres map onto input pixel
// centres, the kernel is stretched by the scale factor when shrinking (so every input
// pixel contributes), taps outside the image are dropped and the rest renormalised.
//
// One CTA per 14x14 output patch.  The CTA computes the patch's horizontal and vertical
// tap tables, resamples the source rows under the patch horizontally into shared memory
// (fp32), then resamples vertically, normalises and stores.  Every product and sum uses
// explicitly rounded fp32 operations, so the pixel and patch-vector forms produce
// identical values.
#include <cuda_bf16.h>

#include "internal.h"

namespace vt {
namespace {

typedef __nv_bfloat16 bf16;

constexpr int kPatchMax = 16;
constexpr int kTapMax = 2 * 2 * kMaxShrink + 4;  // taps of one output pixel at the largest shrink

__device__ unsigned int g_pre_err;

__device__ __forceinline__ float keys_cubic(float x) {
  const float a = -0.5f;
  x = fabsf(x);
  if (x <= 1.f) return __fmaf_rn(__fmul_rn(__fmaf_rn(a + 2.f, x, -(a + 3.f)), x), x, 1.f);
  if (x < 2.f) return __fmul_rn(__fmaf_rn(__fmaf_rn(x - 5.f, x, 8.f), x, -4.f), a);
  return 0.f;
}

// Taps of output index i along one axis: first input index, count, normalised weights.
__device__ void axis_taps(int i, int n_in, int n_out, int* lo_out, int* n_taps, float* w) {
  const float scale = __fdiv_rn(static_cast<float>(n_in), static_cast<float>(n_out));
  const float stretch = fmaxf(scale, 1.f);
  const float support = 2.f * stretch;
  const float c = __fmul_rn(static_cast<float>(i) + 0.5f, scale);
  const int lo = max(static_cast<int>(c - support + 0.5f), 0);
  const int hi = min(static_cast<int>(c + support + 0.5f), n_in);
  const int n = min(hi - lo, kTapMax);
  float sum = 0.f;
  for (int k = 0; k < n; ++k) {
    const float wk = keys_cubic(__fdiv_rn(static_cast<float>(lo + k) + 0.5f - c, stretch));
    w[k] = wk;
    sum = __fadd_rn(sum, wk);
  }
  for (int k = 0; k < n; ++k) w[k] = __fdiv_rn(w[k], sum);
  *lo_out = lo;
  *n_taps = n;
  if (hi - lo > kTapMax) atomicOr(&g_pre_err, 1u);
}

// MODE 0: pixels fp32 [B, 3, gh*p, gw*p].  MODE 1: patch vectors bf16 [B*gh*gw, 3*tp*p*p]
// with tokens in `order`.
template <int MODE>
__global__ void __launch_bounds__(256) preprocess_kernel(const uint8_t* __restrict__ images,
                                                         const PreprocTable tab, void* __restrict__ out,
                                                         int gh, int gw, int patch, int tp, int order,
                                                         int rows_cap) {
  extern __shared__ float rows_h[];  // [rows][patch][3]: source rows resampled along the width
  __shared__ float wy[kPatchMax][kTapMax], wx[kPatchMax][kTapMax];
  __shared__ int ylo[kPatchMax], yn[kPatchMax], xlo[kPatchMax], xn[kPatchMax];

  const int ntok = gh * gw;
  const int row = blockIdx.x;
  const int b = row / ntok, n = row - (row / ntok) * ntok;
  int t, hh, ww;
  token_position(n, gh, gw, order, &t, &hh, &ww);
  const int H0 = tab.src_h[b], W0 = tab.src_w[b];
  const int H1 = gh * patch, W1 = gw * patch;
  const uint8_t* src = images + tab.src_off[b];

  const int tid = threadIdx.x;
  if (tid < patch) axis_taps(hh * patch + tid, H0, H1, &ylo[tid], &yn[tid], wy[tid]);
  else if (tid >= 32 && tid < 32 + patch)
    axis_taps(ww * patch + tid - 32, W0, W1, &xlo[tid - 32], &xn[tid - 32], wx[tid - 32]);
  __syncthreads();

  const int y0 = ylo[0];
  int rows = ylo[patch - 1] + yn[patch - 1] - y0;
  if (rows > rows_cap) {
    if (tid == 0) atomicOr(&g_pre_err, 2u);
    rows = rows_cap;
  }
  const int per_row = patch * 3;
  for (int idx = tid; idx < rows * per_row; idx += blockDim.x) {
    const int r = idx / per_row, rem = idx - r * per_row;
    const int ox = rem / 3, c = rem - ox * 3;
    const uint8_t* s = src + (static_cast<size_t>(y0 + r) * W0 + xlo[ox]) * 3 + c;
    float acc = 0.f;
    for (int k = 0; k < xn[ox]; ++k) acc = __fmaf_rn(wx[ox][k], static_cast<float>(s[3 * k]), acc);
    rows_h[idx] = acc;
  }
  __syncthreads();

  const int pp = patch * patch;
  for (int idx = tid; idx < 3 * pp; idx += blockDim.x) {
    const int c = idx / pp, rem = idx - c * pp;
    const int kh = rem / patch, kw = rem - kh * patch;
    const int r0 = ylo[kh] - y0;
    const int nk = min(yn[kh], rows - r0);
    float acc = 0.f;
    for (int k = 0; k < nk; ++k) acc = __fmaf_rn(wy[kh][k], rows_h[(r0 + k) * per_row + kw * 3 + c], acc);
    const float x = __fdiv_rn(__fsub_rn(__fdiv_rn(acc, 255.f), tab.mean[c]), tab.std[c]);
    if (MODE == 0) {
      float* o = static_cast<float*>(out);
      o[((static_cast<size_t>(b) * 3 + c) * H1 + hh * patch + kh) * W1 + ww * patch + kw] = x;
    } else {
      bf16* o = static_cast<bf16*>(out) + static_cast<size_t>(row) * 3 * tp * pp;
      const bf16 v = __float2bfloat16_rn(x);
      for (int f = 0; f < tp; ++f) o[c * tp * pp + f * pp + rem] = v;
    }
  }
}

}  // namespace

size_t preprocess_rows_bound(int src, int dst, int patch) {
  // rows under one patch: (patch - 1) * scale + 2 * support + 1, plus float slack
  const double scale = static_cast<double>(src) / dst;
  const double stretch = scale > 1.0 ? scale : 1.0;
  const size_t r = static_cast<size_t>((patch - 1) * scale + 4.0 * stretch) + 4;
  return r < static_cast<size_t>(src) ? r : static_cast<size_t>(src);
}

cudaError_t launch_preprocess(const uint8_t* images, const PreprocTable& tab, void* out, int gh, int gw,
                              int patch, int tp, int order, int to_patches, int rows_cap, cudaStream_t stream) {
  if (patch > kPatchMax || tab.count <= 0) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(rows_cap) * patch * 3 * sizeof(float);
  const unsigned blocks = static_cast<unsigned>(tab.count) * gh * gw;
  if (to_patches) {
    cudaFuncSetAttribute(preprocess_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    preprocess_kernel<1><<<blocks, 256, smem, stream>>>(images, tab, out, gh, gw, patch, tp, order, rows_cap);
  } else {
    cudaFuncSetAttribute(preprocess_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    preprocess_kernel<0><<<blocks, 256, smem, stream>>>(images, tab, out, gh, gw, patch, tp, order, rows_cap);
  }
  return cudaGetLastError();
}

unsigned int preprocess_read_clear_error(cudaStream_t stream) {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_pre_err, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return 0;
  cudaStreamSynchronize(stream);
  if (v) {
    cudaMemcpyToSymbolAsync(g_pre_err, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    cudaStreamSynchronize(stream);
  }
  return v;
}

}  // namespace vt
