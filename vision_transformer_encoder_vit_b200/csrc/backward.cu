// Memory-bound kernels of the tower backward: LayerNorm backward with the residual
// gradient added, the per-query delta = rowsum(dO * O) of the attention backward,
// batched 2D transposes (operands of the attention backward, transposed weights), and
// the fold of patch-vector gradients back onto the image (the transpose of the patch
// unfold).
//
// The derivatives are those of the forward of the "MiniMax-M3 Vision" model card
// (Architecture table: pre-LN CLIP-style blocks, Conv3d patch embed with temporal
// patch 2), backpropagated to the image as the differentiable loaders of "v2_loaders -
// Differentiable Vision Tower Loaders (spark2)" do (summary, section 3).
#include <cuda_bf16.h>

#include "internal.h"

namespace vt {
namespace {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    const float2 t = __bfloat1622float2(h);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// dx = dres + (g - mean(g) - xhat * mean(g * xhat)) / sigma with g = dy * gamma, one warp
// per row of 8 * 32 * NV columns; dres may alias dx.
template <int NV>
__global__ void __launch_bounds__(128) layernorm_bwd_warp(const bf16* __restrict__ x, const bf16* __restrict__ gamma,
                                                          const bf16* __restrict__ dy, const bf16* dres, bf16* dx,
                                                          int rows, float eps) {
  constexpr int COLS = 8 * 32 * NV;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const size_t base = static_cast<size_t>(row) * COLS;
  float xv[NV][8], gv[NV][8];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane) * 8;
    unpack8(*reinterpret_cast<const uint4*>(x + base + c), xv[i]);
    float gm[8], d[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(gamma + c)), gm);
    unpack8(*reinterpret_cast<const uint4*>(dy + base + c), d);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      gv[i][e] = d[e] * gm[e];
      s += xv[i][e];
    }
  }
  const float mean = warp_sum(s) * (1.0f / COLS);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float t = xv[i][e] - mean;
      q += t * t;
    }
  const float rstd = rsqrtf(warp_sum(q) * (1.0f / COLS) + eps);
  float sg = 0.f, sgx = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      xv[i][e] = (xv[i][e] - mean) * rstd;  // xhat
      sg += gv[i][e];
      sgx += gv[i][e] * xv[i][e];
    }
  const float mg = warp_sum(sg) * (1.0f / COLS), mgx = warp_sum(sgx) * (1.0f / COLS);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane) * 8;
    float r[8], o[8];
    unpack8(*reinterpret_cast<const uint4*>(dres + base + c), r);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = r[e] + rstd * (gv[i][e] - mg - xv[i][e] * mgx);
    *reinterpret_cast<uint4*>(dx + base + c) = pack8(o);
  }
}

// Any width: one 256-thread block per row, three passes over the row.
__global__ void __launch_bounds__(256) layernorm_bwd_block(const bf16* __restrict__ x, const bf16* __restrict__ gamma,
                                                           const bf16* __restrict__ dy, const bf16* dres, bf16* dx,
                                                           int cols, float eps) {
  __shared__ float red[4][8];
  const size_t base = static_cast<size_t>(blockIdx.x) * cols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto block_sum = [&](float v, int slot) -> float {
    v = warp_sum(v);
    if (lane == 0) red[slot][warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[slot][w];
    return t;
  };
  float s = 0.f;
  for (int c = threadIdx.x; c < cols; c += 256) s += __bfloat162float(x[base + c]);
  const float mean = block_sum(s, 0) / cols;
  float q = 0.f;
  for (int c = threadIdx.x; c < cols; c += 256) {
    const float t = __bfloat162float(x[base + c]) - mean;
    q += t * t;
  }
  const float rstd = rsqrtf(block_sum(q, 1) / cols + eps);
  float sg = 0.f, sgx = 0.f;
  for (int c = threadIdx.x; c < cols; c += 256) {
    const float g = __bfloat162float(dy[base + c]) * __bfloat162float(gamma[c]);
    sg += g;
    sgx += g * (__bfloat162float(x[base + c]) - mean) * rstd;
  }
  const float mg = block_sum(sg, 2) / cols, mgx = block_sum(sgx, 3) / cols;
  for (int c = threadIdx.x; c < cols; c += 256) {
    const float g = __bfloat162float(dy[base + c]) * __bfloat162float(gamma[c]);
    const float xh = (__bfloat162float(x[base + c]) - mean) * rstd;
    dx[base + c] = __float2bfloat16_rn(__bfloat162float(dres[base + c]) + rstd * (g - mg - xh * mgx));
  }
}

// delta[(b*H + h) * ld + n] = sum_d dO[b*N + n, h*D + d] * O[b*N + n, h*D + d]; one
// thread per (token, head).
__global__ void __launch_bounds__(256) attn_delta_kernel(const bf16* __restrict__ dO, const bf16* __restrict__ O,
                                                         float* __restrict__ delta, int B, int N, int H, int D,
                                                         int ld) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long total = static_cast<long>(B) * N * H;
  if (idx >= total) return;
  const int h = static_cast<int>(idx % H);
  const long tok = idx / H;
  const int b = static_cast<int>(tok / N), n = static_cast<int>(tok - static_cast<long>(b) * N);
  const size_t off = static_cast<size_t>(tok) * H * D + static_cast<size_t>(h) * D;
  float s = 0.f;
  for (int d = 0; d < D; d += 8) {
    float a[8], c[8];
    unpack8(*reinterpret_cast<const uint4*>(dO + off + d), a);
    unpack8(*reinterpret_cast<const uint4*>(O + off + d), c);
#pragma unroll
    for (int e = 0; e < 8; ++e) s = fmaf(a[e], c[e], s);
  }
  delta[(static_cast<size_t>(b) * H + h) * ld + n] = s;
}

// Batched transpose: for batch z = (b, h), out[c][r] = in[r][c] for r < R, c < C, with
// in = src + b * in_sb + h * in_sh (row stride in_ld) and out = dst + b * out_sb +
// h * out_sh (row stride out_ld), all in elements.  32x32 tiles through shared memory.
__global__ void __launch_bounds__(256) transpose_kernel(const bf16* __restrict__ src, bf16* __restrict__ dst, int R,
                                                        int C, int H, long in_sb, long in_sh, long in_ld, long out_sb,
                                                        long out_sh, long out_ld) {
  __shared__ bf16 tile[32][34];
  const int z = blockIdx.z, b = z / H, h = z - (z / H) * H;
  const bf16* in = src + b * in_sb + h * in_sh;
  bf16* out = dst + b * out_sb + h * out_sh;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows per pass
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    if (r < R && c < C) tile[i][tx] = in[r * in_ld + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + tx;
    if (r < R && c < C) out[c * out_ld + r] = tile[tx][i];
  }
}

// d_pixels[b, c, y, x] = sum over the tp repeated frames of the patch-vector gradient
// du[row, c*tp*p*p + f*p*p + (y%p)*p + x%p], row = the token of patch (y/p, x/p) in
// `order`.  One thread per pixel.
__global__ void __launch_bounds__(256) patch_fold_kernel(const bf16* __restrict__ du, float* __restrict__ dpx, int B,
                                                         int H, int W, int patch, int tp, int order) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long total = static_cast<long>(B) * 3 * H * W;
  if (idx >= total) return;
  const int xw = static_cast<int>(idx % W);
  const long t1 = idx / W;
  const int yh = static_cast<int>(t1 % H);
  const long t2 = t1 / H;
  const int c = static_cast<int>(t2 % 3);
  const int b = static_cast<int>(t2 / 3);
  const int gh = H / patch, gw = W / patch;
  const int ph = yh / patch, pw = xw / patch, kh = yh - ph * patch, kw = xw - pw * patch;
  int n;
  if (order == ORDER_BLOCK) n = 4 * ((ph >> 1) * (gw >> 1) + (pw >> 1)) + ((ph & 1) << 1) + (pw & 1);
  else n = ph * gw + pw;
  const int pp = patch * patch, K = 3 * tp * pp;
  const bf16* row = du + (static_cast<size_t>(b) * gh * gw + n) * K + c * tp * pp + kh * patch + kw;
  float s = 0.f;
  for (int f = 0; f < tp; ++f) s += __bfloat162float(row[f * pp]);
  dpx[idx] = s;
}

}  // namespace

cudaError_t launch_layernorm_backward(const void* x, const void* gamma, const void* dy, const void* dres, void* dx,
                                      int rows, int cols, float eps, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const bf16 *X = static_cast<const bf16*>(x), *G = static_cast<const bf16*>(gamma),
             *DY = static_cast<const bf16*>(dy), *DR = static_cast<const bf16*>(dres);
  bf16* DX = static_cast<bf16*>(dx);
  const int blocks = (rows + 3) / 4;
  if (cols == 1280) layernorm_bwd_warp<5><<<blocks, 128, 0, stream>>>(X, G, DY, DR, DX, rows, eps);
  else if (cols == 1024) layernorm_bwd_warp<4><<<blocks, 128, 0, stream>>>(X, G, DY, DR, DX, rows, eps);
  else if (cols == 512) layernorm_bwd_warp<2><<<blocks, 128, 0, stream>>>(X, G, DY, DR, DX, rows, eps);
  else if (cols == 256) layernorm_bwd_warp<1><<<blocks, 128, 0, stream>>>(X, G, DY, DR, DX, rows, eps);
  else layernorm_bwd_block<<<rows, 256, 0, stream>>>(X, G, DY, DR, DX, cols, eps);
  return cudaGetLastError();
}

cudaError_t launch_attention_delta(const void* dO, const void* O, float* delta, int B, int N, int H, int D, int ld,
                                   cudaStream_t stream) {
  const long total = static_cast<long>(B) * N * H;
  if (total <= 0) return cudaSuccess;
  if (D % 8) return cudaErrorInvalidValue;
  attn_delta_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
      static_cast<const bf16*>(dO), static_cast<const bf16*>(O), delta, B, N, H, D, ld);
  return cudaGetLastError();
}

cudaError_t launch_transpose(const void* src, void* dst, int B, int H, int R, int C, long in_sb, long in_sh,
                             long in_ld, long out_sb, long out_sh, long out_ld, cudaStream_t stream) {
  if (B <= 0 || H <= 0 || R <= 0 || C <= 0) return cudaSuccess;
  dim3 grid((C + 31) / 32, (R + 31) / 32, B * H);
  transpose_kernel<<<grid, 256, 0, stream>>>(static_cast<const bf16*>(src), static_cast<bf16*>(dst), R, C, H, in_sb,
                                             in_sh, in_ld, out_sb, out_sh, out_ld);
  return cudaGetLastError();
}

cudaError_t launch_patch_fold(const void* du, float* dpixels, int B, int H, int W, int patch, int tp, int order,
                              cudaStream_t stream) {
  const long total = static_cast<long>(B) * 3 * H * W;
  if (total <= 0) return cudaSuccess;
  patch_fold_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(static_cast<const bf16*>(du),
                                                                                     dpixels, B, H, W, patch, tp,
                                                                                     order);
  return cudaGetLastError();
}

}  // namespace vt
