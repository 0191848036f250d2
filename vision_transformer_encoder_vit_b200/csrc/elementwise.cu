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
// q and k are rotated by the 3D RoPE of each token's position: within the axis block
// [off, off + s) of an axis, channels (off + j, off + j + s/2) form pair j, turned by
// the angle pos_axis * theta^(-2j/s).  v is transposed to vt [B*H, D, ld_vt].
//
// Persistent kernel over items (token tile of kPrepTok tokens, (image, head) pair),
// the pair index fastest; each block takes one contiguous, balanced range of items
// and recomputes its tokens' (cos, sin) only when the tile changes.  A block has
// kPrepTok * D / 8 threads, so that each thread owns one task of each kind per item:
//  - q and k (kMode 0: copy, 1: RoPE when every half section is a multiple of 8
//    channels): one pair of 16-byte chunks (channels c..c+7 and their partners) of one
//    token, rotated in registers;
//  - v: one 16-byte chunk staged in shared memory (rows an odd number of words apart,
//    so the column reads fall on distinct banks), then one eight-token run of one vt
//    column written with a 16-byte store.
// The next item's 16-byte loads are issued before the current item's stores.  kMode 2
// (other section widths) rotates q and k one channel pair at a time.
constexpr int kPrepTok = 32;

template <int D, int kMode>
__global__ void __launch_bounds__(kPrepTok * D / 8) attention_prep_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                                                               const bf16* __restrict__ v, bf16* __restrict__ qr,
                                                               bf16* __restrict__ kr, bf16* __restrict__ vt,
                                                               long long BH, int N, int ld_vt,
                                                               const int32_t* __restrict__ pos, int s0, int s1, int s2,
                                                               float theta) {
  constexpr int kThreads = kPrepTok * D / 8, kC8 = D / 8, kPC = D / 16, kHalf = D / 2, kRowWords = D / 2 + 1;
  constexpr int kRuns = kPrepTok / 8;  // eight-token runs of a vt column
  constexpr bool kRope = kMode != 0;
  __shared__ uint32_t vtile[kPrepTok][kRowWords];
  __shared__ __align__(16) float2 cs[kRope ? kPrepTok : 1][kHalf];  // (cos, sin) per token and pair
  __shared__ double freq[kRope ? kHalf : 1];  // theta^(-2j/s) / pi per pair
  __shared__ int freq_axis[kRope ? kHalf : 1];
  __shared__ int chunk_map[kPC];  // first chunk | partner chunk << 8 | first pair << 16
  const int tid = threadIdx.x;
  const long long tiles = (N + kPrepTok - 1) / kPrepTok, items = tiles * BH;
  const long long per = items / gridDim.x, extra = items % gridDim.x;
  const long long it0 = blockIdx.x * per + min(static_cast<long long>(blockIdx.x), extra);
  const long long it1 = it0 + per + (blockIdx.x < extra ? 1 : 0);
  if (it0 >= it1) return;
  if (tid == 0) {
    if (kMode == 1) {
      int n = 0;
      const int sec[3] = {s0, s1, s2};
      for (int a = 0, off = 0; a < 3; off += sec[a], ++a)
        for (int c = 0; c < sec[a] / 16; ++c)
          chunk_map[n++] = (off / 8 + c) | ((off / 8 + sec[a] / 16 + c) << 8) | ((off / 2 + 8 * c) << 16);
    } else {
      for (int c = 0; c < kPC; ++c) chunk_map[c] = 2 * c | ((2 * c + 1) << 8);
    }
  }
  if (kRope) {
    for (int pi = tid; pi < kHalf; pi += kThreads) {
      int axis, j, s;
      if (pi < s0 / 2) {
        axis = 0; j = pi; s = s0;
      } else if (pi < (s0 + s1) / 2) {
        axis = 1; j = pi - s0 / 2; s = s1;
      } else {
        axis = 2; j = pi - (s0 + s1) / 2; s = s2;
      }
      freq[pi] = pow(static_cast<double>(theta), -2.0 * j / s) / 3.141592653589793;
      freq_axis[pi] = axis;
    }
  }
  // This thread's tasks: q/k chunk pair (matrix qm, token qt, chunk pair qc); v chunk
  // (token vt_t, chunk vc); vt run (channel td, tokens 8 * tc ..).
  const int qm = tid >= kThreads / 2, qi = tid - qm * (kThreads / 2), qt = qi / kPC, qc = qi - qt * kPC;
  const int vt_t = tid / kC8, vc = tid - vt_t * kC8;
  const int td = tid / kRuns, tc = tid - td * kRuns;
  const bf16* qsrc = qm ? k : q;
  bf16* qdst = qm ? kr : qr;
  __syncthreads();
  const int cm = chunk_map[qc];
  uint4 na = make_uint4(0, 0, 0, 0), nb = na, nv = na;  // the next item's chunks
  auto load = [&](long long it) {
    const long long tl = it / BH, bh = it - tl * BH;
    const int n0 = static_cast<int>(tl) * kPrepTok, rows = min(kPrepTok, N - n0);
    const size_t row0 = (static_cast<size_t>(bh) * N + n0) * D;
    if (kMode != 2 && qt < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(qsrc + row0 + static_cast<size_t>(qt) * D);
      na = __ldg(src + (cm & 255));
      nb = __ldg(src + ((cm >> 8) & 255));
    }
    if (vt_t < rows) nv = __ldg(reinterpret_cast<const uint4*>(v + row0) + tid);
  };
  load(it0);
  long long table_tile = -1;
  for (long long it = it0; it < it1; ++it) {
    const long long tl = it / BH, bh = it - tl * BH;
    const int n0 = static_cast<int>(tl) * kPrepTok, rows = min(kPrepTok, N - n0);
    const size_t row0 = (static_cast<size_t>(bh) * N + n0) * D;
    __syncthreads();  // the previous item's vt columns and (cos, sin) read
    if (kRope && tl != table_tile) {
      // Angle in half-turns, reduced exactly (in double) to [-1, 1] before the
      // single-precision sincospi: cos and sin within a few 1e-7 of exact.
      for (int e = tid; e < kPrepTok * kHalf; e += kThreads) {
        const int t = e / kHalf, pi = e - t * kHalf;
        if (t < rows) {
          double x = static_cast<double>(pos[static_cast<size_t>(n0 + t) * 3 + freq_axis[pi]]) * freq[pi];
          x -= 2.0 * rint(0.5 * x);
          float sn, c;
          sincospif(static_cast<float>(x), &sn, &c);
          cs[t][pi] = make_float2(c, sn);
        }
      }
      table_tile = tl;
    }
    if (vt_t < rows) {
      uint32_t* w = &vtile[vt_t][4 * vc];
      w[0] = nv.x; w[1] = nv.y; w[2] = nv.z; w[3] = nv.w;
    }
    const uint4 ca = na, cb = nb;
    __syncthreads();
    if (it + 1 < it1) load(it + 1);  // in flight while this item is written
    if (kMode != 2) {
      if (qt < rows) {
        uint4* dst = reinterpret_cast<uint4*>(qdst + row0 + static_cast<size_t>(qt) * D);
        if (kMode == 0) {
          dst[cm & 255] = ca;
          dst[(cm >> 8) & 255] = cb;
        } else {
          const float4* c4 = reinterpret_cast<const float4*>(&cs[qt][cm >> 16]);
          const uint32_t* wa = reinterpret_cast<const uint32_t*>(&ca);
          const uint32_t* wb = reinterpret_cast<const uint32_t*>(&cb);
          uint32_t oa[4], ob[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 r = c4[i];  // (cos, sin) of pairs 2i, 2i+1 of the chunk
            const float2 x = unpack_bf16x2(wa[i]), y = unpack_bf16x2(wb[i]);
            oa[i] = pack_bf16x2(x.x * r.x - y.x * r.y, x.y * r.z - y.y * r.w);
            ob[i] = pack_bf16x2(y.x * r.x + x.x * r.y, y.y * r.z + x.y * r.w);
          }
          dst[cm & 255] = make_uint4(oa[0], oa[1], oa[2], oa[3]);
          dst[(cm >> 8) & 255] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
        }
      }
    } else {
      for (int e = tid; e < 2 * kPrepTok * kHalf; e += kThreads) {
        const int m = e / (kPrepTok * kHalf), r = e - m * (kPrepTok * kHalf);
        const int t = r / kHalf, pi = r - t * kHalf;
        if (t >= rows) continue;
        int c1, s;
        if (pi < s0 / 2) {
          c1 = pi; s = s0;
        } else if (pi < (s0 + s1) / 2) {
          c1 = s0 + pi - s0 / 2; s = s1;
        } else {
          c1 = s0 + s1 + pi - (s0 + s1) / 2; s = s2;
        }
        const int c2 = c1 + s / 2;
        const size_t base = row0 + static_cast<size_t>(t) * D;
        const bf16* src = m ? k : q;
        bf16* dst = m ? kr : qr;
        const float x = __bfloat162float(src[base + c1]), y = __bfloat162float(src[base + c2]);
        const float2 a = cs[t][pi];
        dst[base + c1] = __float2bfloat16_rn(x * a.x - y * a.y);
        dst[base + c2] = __float2bfloat16_rn(y * a.x + x * a.y);
      }
    }
    if (8 * tc < rows) {
      const int t0 = 8 * tc;
      uint32_t x[4];  // tokens t0 .. t0+7 of channel td, two per word
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint16_t lo = reinterpret_cast<const uint16_t*>(&vtile[t0 + 2 * i][0])[td];
        const uint16_t hi = reinterpret_cast<const uint16_t*>(&vtile[t0 + 2 * i + 1][0])[td];
        x[i] = lo | (static_cast<uint32_t>(hi) << 16);
      }
      bf16* dst = vt + (static_cast<size_t>(bh) * D + td) * ld_vt + n0 + t0;
      if (t0 + 8 <= rows) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(x[0], x[1], x[2], x[3]);
      } else {
        uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i < rows - t0) d16[i] = static_cast<uint16_t>(x[i >> 1] >> (16 * (i & 1)));
      }
    }
  }
}

template <int D, int kMode>
cudaError_t launch_prep(const bf16* q, const bf16* k, const bf16* v, bf16* qr, bf16* kr, bf16* vt, long long BH, int N,
                        int ld_vt, const int32_t* pos, const int* sec, float theta, cudaStream_t stream) {
  static int resident = 0;  // blocks of this kernel one SM holds
  if (!resident) {
    int r = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, attention_prep_kernel<D, kMode>, kPrepTok * D / 8, 0);
    resident = r < 1 ? 1 : r;
  }
  const long long items = (N + kPrepTok - 1) / kPrepTok * BH;
  const long long cap = static_cast<long long>(resident) * device_sm_count();
  const unsigned grid = static_cast<unsigned>(items < cap ? items : cap);
  attention_prep_kernel<D, kMode><<<grid, kPrepTok * D / 8, 0, stream>>>(q, k, v, qr, kr, vt, BH, N, ld_vt, pos,
                                                              sec ? sec[0] : 0, sec ? sec[1] : 0, sec ? sec[2] : 0,
                                                              theta);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_prep_d(const bf16* q, const bf16* k, const bf16* v, bf16* qr, bf16* kr, bf16* vt, long long BH,
                          int N, int ld_vt, const int32_t* pos, const int* sec, float theta, cudaStream_t stream) {
  if (!pos) return launch_prep<D, 0>(q, k, v, qr, kr, vt, BH, N, ld_vt, nullptr, nullptr, 0.f, stream);
  if (sec[0] % 16 == 0 && sec[1] % 16 == 0 && sec[2] % 16 == 0)
    return launch_prep<D, 1>(q, k, v, qr, kr, vt, BH, N, ld_vt, pos, sec, theta, stream);
  return launch_prep<D, 2>(q, k, v, qr, kr, vt, BH, N, ld_vt, pos, sec, theta, stream);
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
  const long long BH = static_cast<long long>(B) * H;
  const bf16 *Q = static_cast<const bf16*>(q), *K = static_cast<const bf16*>(k), *V = static_cast<const bf16*>(v);
  bf16 *QR = static_cast<bf16*>(qr), *KR = static_cast<bf16*>(kr), *VT = static_cast<bf16*>(vt);
  switch (D) {
    case 32: return launch_prep_d<32>(Q, K, V, QR, KR, VT, BH, N, ld_vt, pos, sections, theta, stream);
    case 64: return launch_prep_d<64>(Q, K, V, QR, KR, VT, BH, N, ld_vt, pos, sections, theta, stream);
    case 80: return launch_prep_d<80>(Q, K, V, QR, KR, VT, BH, N, ld_vt, pos, sections, theta, stream);
    case 96: return launch_prep_d<96>(Q, K, V, QR, KR, VT, BH, N, ld_vt, pos, sections, theta, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vt
