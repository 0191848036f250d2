// Memory-bound kernels: LayerNorm, patch unfold, row reordering between raster and
// 2x2-block token order, and the RoPE / V-transpose preparation used by the
// stand-alone attention entry point.  Each is a coalesced, vectorised pass; none of
// them is a contraction, so none uses the tensor cores.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ LayerNorm
// y = (x - mean) / sqrt(var + eps) * gamma + beta over each row (pre-LN CLIP-style
// block: norm1 / norm2 of the ViT block in
// "metrale_model_arch/weight_loader/qwen3_vl.rs", load_vision_encoder).  One warp per
// row; a lane holds NV vectors of VEC consecutive bf16 at (i * 32 + lane) * VEC.
// Statistics in fp32, variance from the centred values (two passes over registers).

template <int VEC>
struct VecT;
template <>
struct VecT<8> { typedef uint4 T; };
template <>
struct VecT<4> { typedef uint2 T; };
template <>
struct VecT<2> { typedef uint32_t T; };

template <int VEC>
__device__ __forceinline__ void unpack_vec(typename VecT<VEC>::T u, float* f) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < VEC / 2; ++i) {
    const float2 t = unpack_bf16x2(w[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <int VEC>
__device__ __forceinline__ typename VecT<VEC>::T pack_vec(const float* f) {
  typename VecT<VEC>::T u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < VEC / 2; ++i) w[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
  return u;
}

// The rows stay packed as bf16 in registers (VEC/2 words per vector) and are unpacked
// on the fly in each pass.  A warp walks rows with a stride of all warps of the grid
// (a few rows each, the grid sized to the SMs) and loads its next row while it
// normalises the current one, so that reading and writing overlap in every warp; gamma
// and beta are read through L1, where they stay for all rows of the SM.
template <int VEC, int NV>
__global__ void __launch_bounds__(256, 2) layernorm_warp(const bf16* __restrict__ x, const bf16* __restrict__ gamma,
                                                         const bf16* __restrict__ beta, bf16* __restrict__ y,
                                                         int rows, float eps) {
  typedef typename VecT<VEC>::T V;
  constexpr int COLS = 32 * VEC * NV;
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * (blockDim.x >> 5);
  int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const V* gr = reinterpret_cast<const V*>(gamma);
  const V* br = reinterpret_cast<const V*>(beta);
  V xv[NV];
  {
    const V* xr = reinterpret_cast<const V*>(x + static_cast<size_t>(row) * COLS);
#pragma unroll
    for (int i = 0; i < NV; ++i) xv[i] = xr[i * 32 + lane];
  }
  for (; row < rows; row += stride) {
    const int next = row + stride;
    V xn[NV];
    if (next < rows) {
      const V* xr = reinterpret_cast<const V*>(x + static_cast<size_t>(next) * COLS);
#pragma unroll
      for (int i = 0; i < NV; ++i) xn[i] = xr[i * 32 + lane];
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float f[VEC];
      unpack_vec<VEC>(xv[i], f);
#pragma unroll
      for (int e = 0; e < VEC; ++e) s += f[e];
    }
    const float mean = warp_sum(s) * (1.0f / COLS);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float f[VEC];
      unpack_vec<VEC>(xv[i], f);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float d = f[e] - mean;
        q += d * d;
      }
    }
    const float rstd = rsqrtf(warp_sum(q) * (1.0f / COLS) + eps);
    V* yr = reinterpret_cast<V*>(y + static_cast<size_t>(row) * COLS);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float f[VEC], g[VEC], bb[VEC], o[VEC];
      unpack_vec<VEC>(xv[i], f);
      unpack_vec<VEC>(__ldg(gr + i * 32 + lane), g);
      unpack_vec<VEC>(__ldg(br + i * 32 + lane), bb);
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[e] = (f[e] - mean) * rstd * g[e] + bb[e];
      yr[i * 32 + lane] = pack_vec<VEC>(o);
    }
    if (next < rows) {
#pragma unroll
      for (int i = 0; i < NV; ++i) xv[i] = xn[i];
    }
  }
}

// Any width: one block of 256 threads per row, statistics through shared memory.
__global__ void __launch_bounds__(256) layernorm_block(const bf16* __restrict__ x, const bf16* __restrict__ gamma,
                                                       const bf16* __restrict__ beta, bf16* __restrict__ y,
                                                       int cols, float eps) {
  __shared__ float red[8];
  __shared__ float stat;
  const bf16* xr = x + static_cast<size_t>(blockIdx.x) * cols;
  bf16* yr = y + static_cast<size_t>(blockIdx.x) * cols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float s = 0.f;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) s += __bfloat162float(xr[c]);
  s = warp_sum(s);
  if (lane == 0) red[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < 8; ++i) t += red[i];
    stat = t / cols;
  }
  __syncthreads();
  const float mean = stat;
  float q = 0.f;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    const float d = __bfloat162float(xr[c]) - mean;
    q += d * d;
  }
  q = warp_sum(q);
  __syncthreads();
  if (lane == 0) red[warp] = q;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < 8; ++i) t += red[i];
    stat = rsqrtf(t / cols + eps);
  }
  __syncthreads();
  const float rstd = stat;
  for (int c = threadIdx.x; c < cols; c += blockDim.x)
    yr[c] = __float2bfloat16_rn((__bfloat162float(xr[c]) - mean) * rstd * __bfloat162float(gamma[c]) +
                                __bfloat162float(beta[c]));
}

// -------------------------------------------------------------- patch unfold
// Patch vectors of clips of F frames [B, F, 3, H, W], flattened in (c, t, kh, kw) order
// to match a Conv3d weight [hidden, 3, tp, p, p].  Temporal patch t covers frames
// t*tp .. t*tp+tp-1, the last frame repeated when F is not a multiple of tp; a still
// image is the clip F = 1, its frame repeated tp times ("v2_loaders" findings, section 3:
// temporal dimension padded to 2 by repeating the frame).  One block per token; the
// fp32 pixel is rounded to bf16 (nearest even).
__global__ void __launch_bounds__(256) patch_unfold_kernel(const float* __restrict__ px, bf16* __restrict__ out,
                                                           int F, int H, int W, int patch, int tp, int gt, int gh,
                                                           int gw, int order) {
  const int ntok = gt * gh * gw;
  const int row = blockIdx.x;
  const int b = row / ntok, n = row - (row / ntok) * ntok;
  int t, hh, ww;
  token_position(n, gh, gw, order, &t, &hh, &ww);
  const int pp = patch * patch;
  const int K = 3 * tp * pp;
  bf16* dst = out + static_cast<size_t>(row) * K;
  const float* clip = px + static_cast<size_t>(b) * F * 3 * H * W;
  for (int e = threadIdx.x; e < 3 * pp; e += blockDim.x) {
    const int c = e / pp, rem = e - c * pp;
    const int kh = rem / patch, kw = rem - kh * patch;
    const size_t pix = (static_cast<size_t>(c) * H + hh * patch + kh) * W + ww * patch + kw;
    for (int f = 0; f < tp; ++f) {
      const int frame = min(t * tp + f, F - 1);
      dst[c * tp * pp + f * pp + rem] = __float2bfloat16_rn(clip[static_cast<size_t>(frame) * 3 * H * W + pix]);
    }
  }
}

// Variable-resolution form: one block per packed token; the image comes from the table.
__global__ void __launch_bounds__(256) patch_unfold_varlen_kernel(const float* __restrict__ px,
                                                                  bf16* __restrict__ out, const VarlenTable vl,
                                                                  int patch, int tp) {
  const int row = blockIdx.x;
  const int b = varlen_image(vl, row);
  const int n = row - vl.tok_off[b];
  const int gh = vl.gh[b], gw = vl.gw[b];
  const int H = gh * patch, W = gw * patch;
  int t, hh, ww;
  token_position(n, gh, gw, ORDER_BLOCK, &t, &hh, &ww);
  const int pp = patch * patch;
  const int K = 3 * tp * pp;
  bf16* dst = out + static_cast<size_t>(row) * K;
  const float* img = px + vl.pix_off[b];
  for (int e = threadIdx.x; e < 3 * pp; e += blockDim.x) {
    const int c = e / pp, rem = e - c * pp;
    const int kh = rem / patch, kw = rem - kh * patch;
    const bf16 v = __float2bfloat16_rn(img[(static_cast<size_t>(c) * H + hh * patch + kh) * W + ww * patch + kw]);
    for (int f = 0; f < tp; ++f) dst[c * tp * pp + f * pp + rem] = v;
  }
}

// ------------------------------------------------------------------ reorder
// Moves whole rows between raster order and 2x2-block order (the 2x2 merge of the
// "MiniMax-M3 Vision" model card groups each block's four tokens).
__global__ void __launch_bounds__(256) reorder_rows_kernel(const uint4* __restrict__ in, uint4* __restrict__ out,
                                                           int total_rows, int gh, int gw, int ntok, int vec_per_row,
                                                           int to_block) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= total_rows) return;
  const int b = row / ntok, nb = row - (row / ntok) * ntok;
  int t, hh, ww;
  token_position(nb, gh, gw, ORDER_BLOCK, &t, &hh, &ww);
  const int nr = (t * gh + hh) * gw + ww;
  const size_t base = static_cast<size_t>(b) * ntok;
  const size_t src = base + (to_block ? nr : nb);
  const size_t dst = base + (to_block ? nb : nr);
  for (int i = lane; i < vec_per_row; i += 32)
    out[dst * vec_per_row + i] = in[src * vec_per_row + i];
}

// ------------------------------------------------------ attention preparation
// Rotates q and k by the 3D RoPE of each token's position (pairs (off+j, off+j+s/2)
// of each axis block, angle pos_axis * theta^(-2j/s)) and copies them; one thread per
// (token, pair), looping over batch and heads.
__global__ void __launch_bounds__(256) rope_qk_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                                                      bf16* __restrict__ qr, bf16* __restrict__ kr, int B, int H,
                                                      int N, int D, const int32_t* __restrict__ pos, int s0, int s1,
                                                      int s2, float theta) {
  const int half = D / 2;
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(N) * half) return;
  const int n = static_cast<int>(idx / half);
  const int pi = static_cast<int>(idx - static_cast<long>(n) * half);
  int axis, j, off, s;
  if (pi < s0 / 2) {
    axis = 0; j = pi; off = 0; s = s0;
  } else if (pi < (s0 + s1) / 2) {
    axis = 1; j = pi - s0 / 2; off = s0; s = s1;
  } else {
    axis = 2; j = pi - (s0 + s1) / 2; off = s0 + s1; s = s2;
  }
  const double inv_freq = pow(static_cast<double>(theta), -2.0 * j / s);
  const double ang = static_cast<double>(pos[n * 3 + axis]) * inv_freq;
  double sd, cd;
  sincos(ang, &sd, &cd);
  const float c = static_cast<float>(cd), sn = static_cast<float>(sd);
  const int c1 = off + j, c2 = off + j + s / 2;
  for (int bh = 0; bh < B * H; ++bh) {
    const size_t base = (static_cast<size_t>(bh) * N + n) * D;
    float a = __bfloat162float(q[base + c1]), bb = __bfloat162float(q[base + c2]);
    qr[base + c1] = __float2bfloat16_rn(a * c - bb * sn);
    qr[base + c2] = __float2bfloat16_rn(bb * c + a * sn);
    a = __bfloat162float(k[base + c1]);
    bb = __bfloat162float(k[base + c2]);
    kr[base + c1] = __float2bfloat16_rn(a * c - bb * sn);
    kr[base + c2] = __float2bfloat16_rn(bb * c + a * sn);
  }
}

// v [B*H, N, D] -> vt [B*H, D, ld_vt] through a 64-token shared tile.
__global__ void __launch_bounds__(256) transpose_v_kernel(const bf16* __restrict__ v, bf16* __restrict__ vt, int N,
                                                          int D, int ld_vt) {
  __shared__ bf16 tile[64][128 + 2];
  const int n0 = blockIdx.x * 64;
  const size_t bh = blockIdx.y;
  const bf16* src = v + bh * N * static_cast<size_t>(D);
  for (int e = threadIdx.x; e < 64 * D; e += blockDim.x) {
    const int r = e / D, c = e - (e / D) * D;
    if (n0 + r < N) tile[r][c] = src[static_cast<size_t>(n0 + r) * D + c];
  }
  __syncthreads();
  bf16* dst = vt + bh * D * static_cast<size_t>(ld_vt);
  for (int e = threadIdx.x; e < 64 * D; e += blockDim.x) {
    const int c = e / 64, r = e - (e / 64) * 64;
    if (n0 + r < N) dst[static_cast<size_t>(c) * ld_vt + n0 + r] = tile[r][c];
  }
}

// Plain copy of q or k when no rotation is requested.
__global__ void copy_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, size_t n16) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    out[i] = in[i];
}

}  // namespace

cudaError_t launch_layernorm(const void* x, const void* gamma, const void* beta, void* y, int rows, int cols,
                             float eps, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const bf16* X = static_cast<const bf16*>(x);
  const bf16* G = static_cast<const bf16*>(gamma);
  const bf16* Bt = static_cast<const bf16*>(beta);
  bf16* Y = static_cast<bf16*>(y);
  // 8 warps (rows at a time) per block, at most two blocks per SM
  const int need = (rows + 7) / 8, cap = 2 * device_sm_count();
  const int blocks = need < cap ? need : cap;
  if (cols == 1280) layernorm_warp<8, 5><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else if (cols == 1024) layernorm_warp<8, 4><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else if (cols == 768) layernorm_warp<8, 3><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else if (cols == 512) layernorm_warp<8, 2><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else if (cols == 256) layernorm_warp<8, 1><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else if (cols == 128) layernorm_warp<4, 1><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else if (cols == 64) layernorm_warp<2, 1><<<blocks, 256, 0, stream>>>(X, G, Bt, Y, rows, eps);
  else layernorm_block<<<rows, 256, 0, stream>>>(X, G, Bt, Y, cols, eps);
  return cudaGetLastError();
}

cudaError_t launch_patch_unfold(const float* pixels, void* out, int B, int H, int W, int patch, int tp, int order,
                                cudaStream_t stream) {
  return launch_patch_unfold_frames(pixels, out, B, 1, H, W, patch, tp, order, stream);
}

cudaError_t launch_patch_unfold_frames(const float* pixels, void* out, int B, int F, int H, int W, int patch, int tp,
                                       int order, cudaStream_t stream) {
  const int gh = H / patch, gw = W / patch, gt = (F + tp - 1) / tp;
  const long rows = static_cast<long>(B) * gt * gh * gw;
  if (rows <= 0) return cudaSuccess;
  patch_unfold_kernel<<<static_cast<unsigned>(rows), 256, 0, stream>>>(pixels, static_cast<bf16*>(out), F, H, W,
                                                                       patch, tp, gt, gh, gw, order);
  return cudaGetLastError();
}

cudaError_t launch_patch_unfold_varlen(const float* pixels, void* out, const VarlenTable& vl, int patch, int tp,
                                       cudaStream_t stream) {
  const int rows = vl.tok_off[vl.count];
  if (rows <= 0) return cudaSuccess;
  patch_unfold_varlen_kernel<<<rows, 256, 0, stream>>>(pixels, static_cast<bf16*>(out), vl, patch, tp);
  return cudaGetLastError();
}

cudaError_t launch_reorder_rows(const void* in, void* out, int B, int gt, int gh, int gw, int cols, int to_block,
                                cudaStream_t stream) {
  const int ntok = gt * gh * gw;
  const int rows = B * ntok;
  if (rows <= 0) return cudaSuccess;
  const int blocks = (rows + 7) / 8;
  reorder_rows_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(in), static_cast<uint4*>(out), rows, gh,
                                                  gw, ntok, cols / 8, to_block);
  return cudaGetLastError();
}

cudaError_t launch_attention_prep(const void* q, const void* k, const void* v, void* qr, void* kr, void* vt, int B,
                                  int H, int N, int D, int ld_vt, const int32_t* pos, const int sections[3],
                                  float theta, cudaStream_t stream) {
  if (B <= 0 || H <= 0 || N <= 0) return cudaSuccess;
  if (pos) {
    const long threads = static_cast<long>(N) * (D / 2);
    rope_qk_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<bf16*>(qr), static_cast<bf16*>(kr), B,
        H, N, D, pos, sections[0], sections[1], sections[2], theta);
  } else {
    const size_t n16 = static_cast<size_t>(B) * H * N * D / 8;
    copy_kernel<<<1184, 256, 0, stream>>>(static_cast<const uint4*>(q), static_cast<uint4*>(qr), n16);
    copy_kernel<<<1184, 256, 0, stream>>>(static_cast<const uint4*>(k), static_cast<uint4*>(kr), n16);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((N + 63) / 64, B * H);
  transpose_v_kernel<<<grid, 256, 0, stream>>>(static_cast<const bf16*>(v), static_cast<bf16*>(vt), N, D, ld_vt);
  return cudaGetLastError();
}

}  // namespace vt
