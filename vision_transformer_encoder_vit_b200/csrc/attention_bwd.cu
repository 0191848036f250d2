// Backward of the bidirectional multi-head attention for sm_100a, flash style: the
// probabilities are recomputed tile by tile from q, k and the per-query log-sum-exp the
// forward kept, so no [N, N] buffer exists.  For one image and head, with P the
// probabilities of the scaled scores S = scale q k^T and dO the gradient of the output,
//     dv = P^T dO,   dP = dO v^T,   dS = P * (dP - delta),   delta = rowsum(dO * O),
//     dq = scale dS k,   dk = scale dS^T q,
// and dq, dk are rotated back by the 3D RoPE (the transpose of the forward rotation) and
// written into the [token, 3 * hidden] gradient of the qkv projection.
//
// The operation differentiated is the ViT self-attention of the "MiniMax-M3 Vision"
// model card (Architecture table: 16 heads over hidden 1280, 3D RoPE); the loaders of
// "v2_loaders - Differentiable Vision Tower Loaders (spark2)" (summary, section 3)
// backpropagate through it to the image.
//
// Two kernels, one CTA = 10 warps: warp 0 issues TMA loads, warp 1 owns TMEM and issues
// the MMAs from one thread, warps 2..9 are two groups of four that each own one row per
// thread and split every 64-column step between them (columns 0..31 and 32..63), so two
// warps per SM sub-partition hide each other's latencies.
//  * attn_bwd_dq: one CTA per 128 queries; 64-key steps stream K and V^T.
//        S = Q K_j^T, dP = dO V_j^T  (TMEM, double-buffered)  -> dS (bf16, shared)
//        dQ += dS K_j                (TMEM accumulator)
//  * attn_bwd_dkdv: one CTA per 128 keys (K and v^T staged once); 64-query steps stream
//    Q and dO.
//        S^T = K Q_i^T, dP^T = V dO_i^T                      -> P^T, dS^T (bf16, shared)
//        dV += P^T dO_i, dK += dS^T Q_i
// A tile staged once serves both products that read it: the row-major [64 x D] tiles of
// K, Q and dO are the K-major B operand of the score products and, read MN-major (the
// MMA's B-transpose bit), the B operand of dQ, dK and dV; the [D x 64] tiles of v^T are
// the MN-major B operand of dP and the MN-major A operand of dP^T.  So no transposed copy
// is made and every operand byte crosses from L2 once per step.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

__device__ unsigned int g_attn_bwd_err;

constexpr int kThreads = 320;
constexpr int kCompute = 256;  // threads of the two row groups

__host__ __device__ constexpr uint32_t layout_code(int swizzle_bytes) {
  return swizzle_bytes == 128 ? 2u : swizzle_bytes == 64 ? 4u : 6u;
}

// Head layouts with their RoPE sections (head_dim = s_t + s_h + s_w).
struct Heads80 { static constexpr int D = 80, S0 = 16, S1 = 32, S2 = 32; };
struct Heads32 { static constexpr int D = 32, S0 = 8, S1 = 12, S2 = 12; };

template <int D>
struct BwdShape {
  static constexpr int C0 = D >= 64 ? 64 : D;  // channels of chunk 0
  static constexpr int C1 = D - C0;            // channels of chunk 1
  static constexpr int SW0 = C0 * 2, SW1 = C1 * 2;
  static constexpr uint32_t LAY0 = layout_code(SW0), LAY1 = layout_code(SW1);
  static constexpr int SBO0 = 8 * SW0, SBO1 = 8 * SW1;
  static constexpr int BR = 128;            // rows a CTA owns (queries or keys)
  static constexpr int BS = 64;             // rows streamed per step
  static constexpr int BIG = BR * D * 2;    // [128 x D] row-major tile
  static constexpr int SMALL = BS * D * 2;  // [64 x D] row-major tile
  static constexpr int TR = D * BS * 2;     // [D x 64] tile of v^T
  static constexpr int PS = BR * BS * 2;    // [128 x 64] bf16 tile written by the threads
  static constexpr int BAR_BYTES = 256;
  static constexpr int LIMIT = 232448;
  static constexpr int MAX_STAGES = 6;
  // attn_bwd_dq: fixed Q, dO; per stage K, V^T; dS double-buffered
  static constexpr int DQ_STAGE = SMALL + TR;
  static constexpr int DQ_AVAIL = LIMIT - 1024 - BAR_BYTES - 2 * BIG - 2 * PS;
  static constexpr int DQ_STAGES = DQ_AVAIL / DQ_STAGE > MAX_STAGES ? MAX_STAGES : DQ_AVAIL / DQ_STAGE;
  static constexpr int DQ_SMEM = 1024 + 2 * BIG + DQ_STAGES * DQ_STAGE + 2 * PS + BAR_BYTES;
  // attn_bwd_dkdv: fixed K, V; per stage Q, dO and the 64 queries' log-sum-exp and delta
  // (fp32, in the stage's last 1024-byte block); P^T and dS^T double-buffered
  static constexpr int KV_STATS = 2 * SMALL;  // offset of the statistics in a stage
  static constexpr int KV_STAGE = 2 * SMALL + 1024;
  static constexpr int KV_AVAIL = LIMIT - 1024 - BAR_BYTES - 2 * BIG - 4 * PS;
  static constexpr int KV_STAGES = KV_AVAIL / KV_STAGE > MAX_STAGES ? MAX_STAGES : KV_AVAIL / KV_STAGE;
  static constexpr int KV_SMEM = 1024 + 2 * BIG + KV_STAGES * KV_STAGE + 4 * PS + BAR_BYTES;
  static constexpr int TMEM_COLS = 512;
  static_assert(C0 == 32 || C0 == 64, "chunk 0 width");
  static_assert(C1 == 0 || C1 == 16 || C1 == 32 || C1 == 64, "chunk 1 width");
  static_assert(D % 16 == 0 && D <= 128, "head_dim");
  static_assert(KV_STAGES >= 2 && DQ_STAGES >= 3, "shared memory");
  static_assert(DQ_SMEM <= LIMIT && KV_SMEM <= LIMIT, "shared memory");
  static_assert(BIG % 1024 == 0 && SMALL % 1024 == 0 && TR % 1024 == 0 && (BR * C0 * 2) % 1024 == 0 &&
                    (BS * C0 * 2) % 1024 == 0,
                "1024-byte alignment of swizzled tiles");
};

// Descriptor of K-step ks (16 channels) of a K-major [R x D] tile staged as a C0-wide
// chunk followed by a C1-wide chunk.
template <int D, int R>
__device__ __forceinline__ uint64_t kdesc(uint32_t tile, int ks) {
  using S = BwdShape<D>;
  const int c = ks * 16;
  if (c < S::C0) return smem_desc(tile + c * 2, S::SBO0, S::LAY0);
  return smem_desc(tile + R * S::C0 * 2 + (c - S::C0) * 2, S::SBO1, S::LAY1);
}

// Descriptor of K-step ks (16 columns) of a [rows x 64] tile with 128-byte rows.
__device__ __forceinline__ uint64_t wdesc(uint32_t tile, int ks) { return smem_desc(tile + ks * 32, 1024, 2); }

// Streamed [64 x D] row-major tiles (K in dq; Q and dO in dk/dv) are staged as D/16
// chunks of [64 rows x 16 channels], 32-byte swizzled, 2048 bytes each.  Read K-major
// (score products, K = channels), K-step ks is chunk ks with 8-row stride 256.  Read
// MN-major (gradient products, K = the 64 rows, N = the D channels), K-step ks starts 16
// rows down (512 bytes) and one descriptor spans all D channels: N advances chunk by
// chunk (leading byte offset 2048), so each K-step is a single N = D product.
constexpr int kChunk = 64 * 32;
__device__ __forceinline__ uint64_t kdesc32(uint32_t tile, int ks) { return smem_desc(tile + ks * kChunk, 256, 6); }
__device__ __forceinline__ uint64_t mndesc32(uint32_t tile, int ks) {
  const uint64_t d = smem_desc(tile + ks * 16 * 32, 256, 6);
  return (d & ~(static_cast<uint64_t>(0x3FFF) << 16)) | (static_cast<uint64_t>(kChunk >> 4) << 16);
}

// A [D x 64] tile of v^T with 128-byte rows, read as an MN-major operand (N = 64 keys
// along a row, K = channels down the rows): 16 rows per K-step.
__device__ __forceinline__ uint64_t vtdesc(uint32_t tile, int ks) { return smem_desc(tile + ks * 2048, 1024, 2); }

// v^T of a CTA's 128 keys staged as two [D x 64] boxes (128-byte rows: 64 keys of one
// channel), read as the MN-major A operand V (M = the 128 keys along the rows, K = the
// channels down the rows): 16 rows per K-step, the second 64 keys one box further
// (leading byte offset = one box).
template <int D>
__device__ __forceinline__ uint64_t vadesc(uint32_t tile, int ks) {
  const uint64_t d = smem_desc(tile + ks * 2048, 1024, 2);
  return (d & ~(static_cast<uint64_t>(0x3FFF) << 16)) | (static_cast<uint64_t>((D * 128) >> 4) << 16);
}

// Instruction descriptor with the A operand MN-major (bit 15).
__host__ __device__ constexpr uint32_t idesc_amn(int M, int N) { return idesc_bf16_f32(M, N) | (1u << 15); }

// Instruction descriptor with the B operand MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_bmn(int M, int N) { return idesc_bf16_f32(M, N) | (1u << 16); }

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > VT_WAIT_LIMIT_NS) {
      atomicOr(&g_attn_bwd_err, VT_DEVERR_TIMEOUT);
      return;
    }
  }
}

// The transpose of one rotation block: (a, b) rotated by -phi.
template <int OFF, int S>
__device__ __forceinline__ void unrope_block(float* v, const float2* tab_axis_pos) {
#pragma unroll
  for (int j = 0; j < S / 2; ++j) {
    const float2 cs = tab_axis_pos[j];
    const float a = v[OFF + j], b = v[OFF + j + S / 2];
    v[OFF + j] = a * cs.x + b * cs.y;
    v[OFF + j + S / 2] = b * cs.x - a * cs.y;
  }
}

template <class HL>
__device__ __forceinline__ void unrope(float* v, const AttnBwdParams& p, int n) {
  if (!p.rope) return;
  int tp, hp, wp;
  token_position(n, p.gh, p.gw, p.order, &tp, &hp, &wp);
  const float2* tab = p.rope_tab;
  unrope_block<0, HL::S0>(v, tab + static_cast<size_t>(0 * kRopeMaxPos + tp) * kRopePairs);
  unrope_block<HL::S0, HL::S1>(v, tab + static_cast<size_t>(1 * kRopeMaxPos + hp) * kRopePairs);
  unrope_block<HL::S0 + HL::S1, HL::S2>(v, tab + static_cast<size_t>(2 * kRopeMaxPos + wp) * kRopePairs);
}

// Untiled bulk copy global -> shared of `bytes` (a multiple of 16; both addresses 16-byte
// aligned), completion counted on `bar`.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Writes 8 bf16 values to 16-byte chunk `cc` of row r of a 128-byte-swizzled tile.
__device__ __forceinline__ void store_sw128(uint8_t* tile, int r, int cc, const float* v8) {
  *reinterpret_cast<uint4*>(tile + r * 128 + ((cc ^ (r & 7)) << 4)) = pack_bf16x8(v8);
}

// ----------------------------------------------------------------- dq kernel

template <class HL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq(const __grid_constant__ CUtensorMap tmQ0, const __grid_constant__ CUtensorMap tmQ1,
                const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                const __grid_constant__ CUtensorMap tmK16, const __grid_constant__ CUtensorMap tmVT,
                const AttnBwdParams p) {
  constexpr int D = HL::D;
  using S = BwdShape<D>;
  constexpr int ST = S::DQ_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + S::BIG;
  uint8_t* sStage = sdO + S::BIG;  // per stage: K [64 x D], V^T [D x 64]
  uint8_t* sdS = sStage + ST * S::DQ_STAGE;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sdS + 2 * S::PS);
  uint64_t* fixed_full = bar;
  uint64_t* kv_full = bar + 1;
  uint64_t* kv_empty = kv_full + ST;
  uint64_t* s_full = kv_empty + ST;  // [2]
  uint64_t* s_free = s_full + 2;
  uint64_t* ds_full = s_free + 2;
  uint64_t* dq_done = ds_full + 2;
  uint64_t* drain = dq_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* armed = const_cast<int*>(abort_flag + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = p.N, bh = b * p.H + h;
  const int nk = (N + S::BS - 1) / S::BS;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      armed[s] = -1;
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&s_full[u], 1);
      mbar_init(&s_free[u], kCompute);
      mbar_init(&ds_full[u], kCompute);
      mbar_init(&dq_done[u], 1);
    }
    mbar_init(drain, 1);
    armed[ST] = -1;
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(&g_attn_bwd_err) != 0) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort_flag != 0;

  if (!skip && warp == 0) {
    if (lane == 0) {
      const int q_row = bh * N + qt * S::BR;
      const int o_row = b * N + qt * S::BR;
      mbar_arrive_expect_tx(fixed_full, 2 * S::BIG);
      tma_load_2d(sQ, &tmQ0, fixed_full, 0, q_row);
      if (S::C1) tma_load_2d(sQ + S::BR * S::C0 * 2, &tmQ1, fixed_full, S::C0, q_row);
      tma_load_2d(sdO, &tmO0, fixed_full, h * D, o_row);
      if (S::C1) tma_load_2d(sdO + S::BR * S::C0 * 2, &tmO1, fixed_full, h * D + S::C0, o_row);
      armed[ST] = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j % ST;
        const uint32_t ph = (j / ST) & 1;
        if (!mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, &g_attn_bwd_err)) break;
        uint8_t* sK = sStage + s * S::DQ_STAGE;
        uint8_t* sVT = sK + S::SMALL;
        const int k_row = bh * N + j * S::BS;
        mbar_arrive_expect_tx(&kv_full[s], S::DQ_STAGE);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) tma_load_2d(sK + c * kChunk, &tmK16, &kv_full[s], c * 16, k_row);
        tma_load_2d(sVT, &tmVT, &kv_full[s], j * S::BS, bh * D);
        armed[s] = static_cast<int>(ph);
      }
      if (*abort_flag) {
        if (armed[ST] >= 0) drain_wait(fixed_full, 0);
        for (int s = 0; s < ST; ++s)
          if (armed[s] >= 0) drain_wait(&kv_full[s], static_cast<uint32_t>(armed[s]));
      }
    }
  } else if (!skip && warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, S::BS);
      constexpr uint32_t idesc_p = idesc_bmn(128, S::BS);
      constexpr uint32_t idesc_q = idesc_bmn(128, D);
      bool issued = false;
      bool ok = mbar_wait(fixed_full, 0, abort_flag, &g_attn_bwd_err);
      // dQ += dS_i K_i, K_i read MN-major from its row-major tile (channel chunks)
      auto issue_dq = [&](int i) -> bool {
        const int u = i & 1;
        if (!mbar_wait(&ds_full[u], (i >> 1) & 1, abort_flag, &g_attn_bwd_err)) return false;
        tc_fence_after();
        const uint32_t a = smem_u32(sdS + u * S::PS);
        const uint32_t kk = smem_u32(sStage + (i % ST) * S::DQ_STAGE);
#pragma unroll
        for (int ks = 0; ks < S::BS / 16; ++ks) {
          const uint32_t acc = (i > 0 || ks > 0) ? 1u : 0u;
          umma_bf16(tmem + 256, wdesc(a, ks), mndesc32(kk, ks), idesc_q, acc);
        }
        umma_commit(&dq_done[u]);
        umma_commit(&kv_empty[i % ST]);
        return true;
      };
      for (int j = 0; ok && j < nk; ++j) {
        const int s = j % ST, u = j & 1;
        if (!mbar_wait(&kv_full[s], (j / ST) & 1, abort_flag, &g_attn_bwd_err)) {
          ok = false;
          break;
        }
        if (j >= 2 && !mbar_wait(&s_free[u], ((j - 2) >> 1) & 1, abort_flag, &g_attn_bwd_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kq = smem_u32(sQ), kd = smem_u32(sdO);
        const uint32_t kk = smem_u32(sStage + s * S::DQ_STAGE), kvt = kk + S::SMALL;
        // the two products accumulate into different TMEM columns: interleave their K-steps
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          umma_bf16(tmem + u * 128, kdesc<D, 128>(kq, ks), kdesc32(kk, ks), idesc_s, ks > 0 ? 1u : 0u);
          umma_bf16(tmem + u * 128 + 64, kdesc<D, 128>(kd, ks), vtdesc(kvt, ks), idesc_p, ks > 0 ? 1u : 0u);
        }
        issued = true;
        umma_commit(&s_full[u]);
        if (j >= 1) ok = issue_dq(j - 1);
      }
      if (ok) ok = issue_dq(nk - 1);
      if (*abort_flag && issued) {
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (!skip) {
    // --------------------------- one query row per thread, half of each step's columns
    const int grp = (warp - 2) >> 2;  // columns [32 grp, 32 grp + 32) of every step
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int n = qt * S::BR + r;
    const bool row_ok = n < N;
    const float sl2 = p.scale * 1.4426950408889634f;
    const float lse = row_ok ? p.lse[static_cast<size_t>(bh) * p.ld_stats + n] : 0.f;
    const float dlt = row_ok ? p.delta[static_cast<size_t>(bh) * p.ld_stats + n] : 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int u = j & 1;
      if (!mbar_wait(&s_full[u], (j >> 1) & 1, abort_flag, &g_attn_bwd_err)) {
        ok = false;
        break;
      }
      if (j >= 2 && !mbar_wait(&dq_done[u], ((j - 2) >> 1) & 1, abort_flag, &g_attn_bwd_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* ds_tile = sdS + u * S::PS;
      {
        const int c0 = grp * 32;
        uint32_t sr[32], pr[32];
        tmem_ld32(tmem + lane_off + u * 128 + c0, sr);
        tmem_ld32(tmem + lane_off + u * 128 + 64 + c0, pr);
        tmem_ld_wait();
        float ds[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool ok_k = row_ok && (j * S::BS + c0 + i) < N;
          const float pv = fast_exp2(fmaf(__uint_as_float(sr[i]), sl2, -lse));
          ds[i] = ok_k ? pv * (__uint_as_float(pr[i]) - dlt) : 0.f;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) store_sw128(ds_tile, r, c0 / 8 + g, ds + 8 * g);
      }
      tc_fence_before();
      mbar_arrive(&s_free[u]);
      fence_proxy_async_smem();
      mbar_arrive(&ds_full[u]);
    }
    if (ok) ok = mbar_wait(&dq_done[(nk - 1) & 1], ((nk - 1) >> 1) & 1, abort_flag, &g_attn_bwd_err);
    if (ok && grp == 0) {
      tc_fence_after();
      float v[D];
      load_cols<D>(tmem + lane_off + 256, v);
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < D; ++i) v[i] *= p.scale;
        unrope<HL>(v, p, n);
        bf16* dst = static_cast<bf16*>(p.dqkv) + (static_cast<size_t>(b) * N + n) * p.ld_dqkv + h * D;
#pragma unroll
        for (int g = 0; g < D / 8; ++g) reinterpret_cast<uint4*>(dst)[g] = pack_bf16x8(v + 8 * g);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

// --------------------------------------------------------------- dk, dv kernel

template <class HL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv(const __grid_constant__ CUtensorMap tmK0, const __grid_constant__ CUtensorMap tmK1,
                  const __grid_constant__ CUtensorMap tmVT, const __grid_constant__ CUtensorMap tmQ16,
                  const __grid_constant__ CUtensorMap tmO16,
                  const AttnBwdParams p) {
  constexpr int D = HL::D;
  using S = BwdShape<D>;
  constexpr int ST = S::KV_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sVT = sK + S::BIG;              // v^T of this CTA's keys: two [D x 64] boxes
  uint8_t* sStage = sVT + S::BIG;          // per stage: Q [64 x D], dO [64 x D]
  uint8_t* sP = sStage + ST * S::KV_STAGE;  // [2] P^T tiles, then [2] dS^T tiles
  uint8_t* sdS = sP + 2 * S::PS;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sdS + 2 * S::PS);
  uint64_t* fixed_full = bar;
  uint64_t* st_full = bar + 1;
  uint64_t* st_empty = st_full + ST;
  uint64_t* s_full = st_empty + ST;  // [2]
  uint64_t* s_free = s_full + 2;
  uint64_t* pd_full = s_free + 2;
  uint64_t* pd_done = pd_full + 2;
  uint64_t* drain = pd_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* armed = const_cast<int*>(abort_flag + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = p.N, bh = b * p.H + h;
  const int nq = (N + S::BS - 1) / S::BS;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
      armed[s] = -1;
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&s_full[u], 1);
      mbar_init(&s_free[u], kCompute);
      mbar_init(&pd_full[u], kCompute);
      mbar_init(&pd_done[u], 1);
    }
    mbar_init(drain, 1);
    armed[ST] = -1;
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(&g_attn_bwd_err) != 0) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort_flag != 0;

  if (!skip && warp == 0) {
    if (lane == 0) {
      const int k_row = bh * N + kt * S::BR;
      mbar_arrive_expect_tx(fixed_full, 2 * S::BIG);
      tma_load_2d(sK, &tmK0, fixed_full, 0, k_row);
      if (S::C1) tma_load_2d(sK + S::BR * S::C0 * 2, &tmK1, fixed_full, S::C0, k_row);
      tma_load_2d(sVT, &tmVT, fixed_full, kt * S::BR, bh * D);
      tma_load_2d(sVT + D * 128, &tmVT, fixed_full, kt * S::BR + 64, bh * D);
      armed[ST] = 0;
      for (int i = 0; i < nq; ++i) {
        const int s = i % ST;
        const uint32_t ph = (i / ST) & 1;
        if (!mbar_wait(&st_empty[s], ph ^ 1u, abort_flag, &g_attn_bwd_err)) break;
        uint8_t* sQ = sStage + s * S::KV_STAGE;
        uint8_t* sdO = sQ + S::SMALL;
        const int q_row = bh * N + i * S::BS;
        const int o_row = b * N + i * S::BS;
        const size_t st0 = static_cast<size_t>(bh) * p.ld_stats + i * S::BS;
        mbar_arrive_expect_tx(&st_full[s], 2 * S::SMALL + 2 * S::BS * 4);
        bulk_load(sQ + S::KV_STATS, p.lse + st0, S::BS * 4, &st_full[s]);
        bulk_load(sQ + S::KV_STATS + S::BS * 4, p.delta + st0, S::BS * 4, &st_full[s]);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          tma_load_2d(sQ + c * kChunk, &tmQ16, &st_full[s], c * 16, q_row);
          tma_load_2d(sdO + c * kChunk, &tmO16, &st_full[s], h * D + c * 16, o_row);
        }
        armed[s] = static_cast<int>(ph);
      }
      if (*abort_flag) {
        if (armed[ST] >= 0) drain_wait(fixed_full, 0);
        for (int s = 0; s < ST; ++s)
          if (armed[s] >= 0) drain_wait(&st_full[s], static_cast<uint32_t>(armed[s]));
      }
    }
  } else if (!skip && warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, S::BS);
      constexpr uint32_t idesc_o = idesc_bmn(128, D);
      constexpr uint32_t idesc_vs = idesc_amn(128, S::BS);  // dP^T = V dO^T with V read MN-major
      bool issued = false;
      bool ok = mbar_wait(fixed_full, 0, abort_flag, &g_attn_bwd_err);
      // dV += P^T_i dO_i, dK += dS^T_i Q_i; dO_i and Q_i read MN-major (channel chunks)
      auto issue_kv = [&](int i) -> bool {
        const int u = i & 1;
        if (!mbar_wait(&pd_full[u], (i >> 1) & 1, abort_flag, &g_attn_bwd_err)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(sP + u * S::PS), da = smem_u32(sdS + u * S::PS);
        const uint32_t kq = smem_u32(sStage + (i % ST) * S::KV_STAGE), ko = kq + S::SMALL;
#pragma unroll
        for (int ks = 0; ks < S::BS / 16; ++ks) {
          const uint32_t acc = (i > 0 || ks > 0) ? 1u : 0u;
          umma_bf16(tmem + 256, wdesc(pa, ks), mndesc32(ko, ks), idesc_o, acc);
          umma_bf16(tmem + 384, wdesc(da, ks), mndesc32(kq, ks), idesc_o, acc);
        }
        umma_commit(&pd_done[u]);
        umma_commit(&st_empty[i % ST]);
        return true;
      };
      for (int i = 0; ok && i < nq; ++i) {
        const int s = i % ST, u = i & 1;
        if (!mbar_wait(&st_full[s], (i / ST) & 1, abort_flag, &g_attn_bwd_err)) {
          ok = false;
          break;
        }
        if (i >= 2 && !mbar_wait(&s_free[u], ((i - 2) >> 1) & 1, abort_flag, &g_attn_bwd_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kk = smem_u32(sK), kv = smem_u32(sVT);
        const uint32_t kq = smem_u32(sStage + s * S::KV_STAGE), ko = kq + S::SMALL;
        // the two products accumulate into different TMEM columns: interleave their K-steps
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          umma_bf16(tmem + u * 128, kdesc<D, 128>(kk, ks), kdesc32(kq, ks), idesc_s, ks > 0 ? 1u : 0u);
          umma_bf16(tmem + u * 128 + 64, vadesc<D>(kv, ks), kdesc32(ko, ks), idesc_vs, ks > 0 ? 1u : 0u);
        }
        issued = true;
        umma_commit(&s_full[u]);
        if (i >= 1) ok = issue_kv(i - 1);
      }
      if (ok) ok = issue_kv(nq - 1);
      if (*abort_flag && issued) {
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (!skip) {
    // ----------------------------- one key row per thread, half of each step's columns
    const int grp = (warp - 2) >> 2;  // columns [32 grp, 32 grp + 32) of every step
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int n = kt * S::BR + r;
    const bool row_ok = n < N;
    const float sl2 = p.scale * 1.4426950408889634f;
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int u = i & 1;
      if (!mbar_wait(&s_full[u], (i >> 1) & 1, abort_flag, &g_attn_bwd_err)) {
        ok = false;
        break;
      }
      if (i >= 2 && !mbar_wait(&pd_done[u], ((i - 2) >> 1) & 1, abort_flag, &g_attn_bwd_err)) {
        ok = false;
        break;
      }
      // the step's statistics arrived with its stage (that phase cannot advance before
      // this step's gradient products, which wait for these threads)
      if (!mbar_wait(&st_full[i % ST], (i / ST) & 1, abort_flag, &g_attn_bwd_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* stats = reinterpret_cast<const float*>(sStage + (i % ST) * S::KV_STAGE + S::KV_STATS);
      uint8_t* p_tile = sP + u * S::PS;
      uint8_t* d_tile = sdS + u * S::PS;
      {
        const int c0 = grp * 32;
        uint32_t sr[32], pr[32];
        tmem_ld32(tmem + lane_off + u * 128 + c0, sr);
        tmem_ld32(tmem + lane_off + u * 128 + 64 + c0, pr);
        const int q0 = i * S::BS + c0;  // first query of this chunk
        float lq[32], dq[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 a = reinterpret_cast<const float4*>(stats + c0)[g];
          const float4 c = reinterpret_cast<const float4*>(stats + S::BS + c0)[g];
          lq[4 * g] = a.x, lq[4 * g + 1] = a.y, lq[4 * g + 2] = a.z, lq[4 * g + 3] = a.w;
          dq[4 * g] = c.x, dq[4 * g + 1] = c.y, dq[4 * g + 2] = c.z, dq[4 * g + 3] = c.w;
        }
        tmem_ld_wait();
        float pv[32], ds[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const bool ok_q = row_ok && (q0 + k) < N;
          const float e = fast_exp2(fmaf(__uint_as_float(sr[k]), sl2, -lq[k]));
          pv[k] = ok_q ? e : 0.f;
          ds[k] = ok_q ? e * (__uint_as_float(pr[k]) - dq[k]) : 0.f;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          store_sw128(p_tile, r, c0 / 8 + g, pv + 8 * g);
          store_sw128(d_tile, r, c0 / 8 + g, ds + 8 * g);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[u]);
      fence_proxy_async_smem();
      mbar_arrive(&pd_full[u]);
    }
    if (ok) ok = mbar_wait(&pd_done[(nq - 1) & 1], ((nq - 1) >> 1) & 1, abort_flag, &g_attn_bwd_err);
    if (ok) {
      tc_fence_after();
      const int width = p.H * D;
      bf16* row = static_cast<bf16*>(p.dqkv) + (static_cast<size_t>(b) * N + n) * p.ld_dqkv;
      if (grp == 0) {  // dK
        float v[D];
        load_cols<D>(tmem + lane_off + 384, v);
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < D; ++c) v[c] *= p.scale;
          unrope<HL>(v, p, n);
          bf16* dst = row + width + h * D;
#pragma unroll
          for (int g = 0; g < D / 8; ++g) reinterpret_cast<uint4*>(dst)[g] = pack_bf16x8(v + 8 * g);
        }
      }
      if (grp == 1) {  // dV
        float v[D];
        load_cols<D>(tmem + lane_off + 256, v);
        if (row_ok) {
          bf16* dst = row + 2 * width + h * D;
#pragma unroll
          for (int g = 0; g < D / 8; ++g) reinterpret_cast<uint4*>(dst)[g] = pack_bf16x8(v + 8 * g);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

template <class HL>
cudaError_t launch_bwd(const AttnBwdParams& p, cudaStream_t stream) {
  constexpr int D = HL::D;
  using S = BwdShape<D>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq<HL>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::DQ_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dkdv<HL>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::KV_SMEM);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const uint64_t rows = static_cast<uint64_t>(p.B) * p.H * p.N;  // rows of q, k, v [B, H, N, D]
  const uint64_t tok = static_cast<uint64_t>(p.B) * p.N;          // rows of dO [B * N, H * D]
  const uint64_t trows = static_cast<uint64_t>(p.B) * p.H * D;    // rows of v^T [B, H, D, ld]
  CUtensorMap q0_128, q1_128, o0_128, o1_128, q16, o16, k16, k0_128, k1_128, vT;
  auto mk = [&](CUtensorMap* m, const void* base, uint64_t r, uint64_t ld, int box_rows, int col0_width, int sw) {
    return make_tmap_2d(m, base, r, ld, ld, box_rows, col0_width, sw);
  };
  bool ok = true;
  const int C0 = S::C0, C1 = S::C1;
  ok = ok && mk(&q0_128, p.q, rows, D, 128, C0, S::SW0) && mk(&q16, p.q, rows, D, 64, 16, 32);
  ok = ok && mk(&k0_128, p.k, rows, D, 128, C0, S::SW0) && mk(&k16, p.k, rows, D, 64, 16, 32);
  ok = ok && make_tmap_2d(&o0_128, p.dO, tok, static_cast<uint64_t>(p.H) * D, static_cast<uint64_t>(p.H) * D, 128,
                          C0, S::SW0);
  ok = ok && make_tmap_2d(&o16, p.dO, tok, static_cast<uint64_t>(p.H) * D, static_cast<uint64_t>(p.H) * D, 64, 16,
                          32);
  if (C1) {
    ok = ok && mk(&q1_128, p.q, rows, D, 128, C1, S::SW1);
    ok = ok && mk(&k1_128, p.k, rows, D, 128, C1, S::SW1);
    ok = ok && make_tmap_2d(&o1_128, p.dO, tok, static_cast<uint64_t>(p.H) * D, static_cast<uint64_t>(p.H) * D, 128,
                            C1, S::SW1);

  } else {
    q1_128 = q0_128, k1_128 = k0_128, o1_128 = o0_128;
  }
  // v^T: [B*H*D rows, N columns] with row stride ld; columns past N read as zero, so
  // padding never enters an MMA.
  ok = ok && make_tmap_2d(&vT, p.vt, trows, p.N, p.ld, D, 64, 128);
  if (!ok) return cudaErrorInvalidValue;
  dim3 grid((p.N + S::BR - 1) / S::BR, p.H, p.B);
  attn_bwd_dq<HL><<<grid, kThreads, S::DQ_SMEM, stream>>>(q0_128, q1_128, o0_128, o1_128, k16, vT, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv<HL><<<grid, kThreads, S::KV_SMEM, stream>>>(k0_128, k1_128, vT, q16, o16, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_backward(const AttnBwdParams& p, cudaStream_t stream) {
  if (p.B <= 0 || p.H <= 0 || p.N <= 0) return cudaSuccess;
  if (p.D == 80 && (!p.rope || (p.sections[0] == 16 && p.sections[1] == 32 && p.sections[2] == 32)))
    return launch_bwd<Heads80>(p, stream);
  if (p.D == 32 && (!p.rope || (p.sections[0] == 8 && p.sections[1] == 12 && p.sections[2] == 12)))
    return launch_bwd<Heads32>(p, stream);
  return cudaErrorNotSupported;
}

unsigned int attention_bwd_read_clear_error(cudaStream_t stream) {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_attn_bwd_err, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return 0;
  cudaStreamSynchronize(stream);
  if (v) {
    cudaMemcpyToSymbolAsync(g_attn_bwd_err, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    cudaStreamSynchronize(stream);
  }
  return v;
}

}  // namespace vt
