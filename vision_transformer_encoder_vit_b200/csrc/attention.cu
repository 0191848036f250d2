// Bidirectional (non-causal) multi-head attention for sm_100a, flash style:
// O_h = softmax(q_h k_h^T * scale) v_h per image and head, computed for two 128-row
// query tiles per CTA while 128-key tiles stream through a TMA ring.  No [N, N]
// buffer exists anywhere; memory traffic is q, k, v in and o out.
//
// The operation is the ViT self-attention of the "MiniMax-M3 Vision" model card
// (Architecture table: 16 heads over hidden 1280).  The loader page
// "spark_model/layers/vision_encoder/enc_impl/init.rs" (VisionScratch and the doc
// comment of CEILING_MAX_PATCHES) builds the full [seq, seq] score matrix per head and
// notes that larger images need tiled attention; this kernel is that tiled form.
//
// The grid is persistent: at most one CTA per SM, each walking work items (a pair of
// query tiles of one head of one image) with a stride of the grid size, so barrier
// setup and TMEM allocation happen once per SM and the next item's first score
// products run while the current item's last softmax and output are still in flight.
//
// CTA = 10 warps.  Warp 0 issues TMA loads (both Q tiles of an item, then K and V^T
// tiles shared by the two query tiles).  Warp 1 allocates TMEM and issues the MMAs from one
// thread; for key tile j and query tile t in {0, 1}:
//     S_t = Q_t K_j^T         -> TMEM columns [256 t, 256 t + 128)        (fp32)
//     O_t += P_t V_j          -> TMEM columns [256 t + 128, 256 t + 128 + D)
// Warps 2..5 run the online softmax of query tile 0 and warps 6..9 that of query tile
// 1 (one thread per query row): load S_t from TMEM, exponentiate against a lazily
// updated running maximum, write P_t (bf16) into a 128-byte-swizzled shared tile for
// the next MMA, rescale O_t in TMEM only when the maximum grows by more than 2^8, and
// finally write O_t / l.  Two softmax warps per SM sub-partition hide each other's
// latencies, and each K/V tile feeds twice the MMA work of a one-tile CTA.
//
// Operand layouts: q, k are [B, H, N, D] (D contiguous), used K-major; v is given
// transposed, vt [B, H, D, ld_vt], so that V_j^T is K-major too.  A head of 80
// channels is staged as a 64-channel chunk with 128-byte swizzle plus a 16-channel
// chunk with 32-byte swizzle, so no padding is computed.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

__device__ unsigned int g_attn_err;

constexpr int kThreads = 320;

__host__ __device__ constexpr uint32_t layout_code(int swizzle_bytes) {
  return swizzle_bytes == 128 ? 2u : swizzle_bytes == 64 ? 4u : 6u;
}

template <int D>
struct AttnShape {
  static constexpr int BM = 128;  // query rows per tile (two tiles per CTA)
  static constexpr int BN = 128;  // keys per tile
  static constexpr int C0 = D >= 64 ? 64 : D;  // channels of chunk 0
  static constexpr int C1 = D - C0;            // channels of chunk 1 (0 if none)
  static constexpr int SW0 = C0 * 2, SW1 = C1 * 2;  // row bytes = swizzle span
  static constexpr uint32_t LAY0 = layout_code(SW0), LAY1 = layout_code(SW1);
  static constexpr int SBO0 = 8 * SW0, SBO1 = 8 * SW1;
  static constexpr int Q_BYTES = BM * D * 2;  // one query tile
  static constexpr int Q1_OFF = BM * C0 * 2;
  static constexpr int K_BYTES = BN * D * 2;
  static constexpr int K1_OFF = BN * C0 * 2;
  static constexpr int V_BYTES = D * BN * 2;  // two [D x 64] boxes
  static constexpr int V1_OFF = D * 64 * 2;
  static constexpr int KV_BYTES = K_BYTES + V_BYTES;
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int BAR_BYTES = 256;
  static constexpr int AVAIL = 232448 - 1024 - BAR_BYTES - 2 * Q_BYTES - 2 * P_BYTES;
  static constexpr int STAGES = AVAIL / KV_BYTES > 4 ? 4 : AVAIL / KV_BYTES;
  static constexpr int SMEM_BYTES = 1024 + 2 * Q_BYTES + STAGES * KV_BYTES + 2 * P_BYTES + BAR_BYTES;
  static constexpr int TMEM_COLS = 512;
  static_assert(C0 == 16 || C0 == 32 || C0 == 64, "chunk 0 width");
  static_assert(C1 == 0 || C1 == 16 || C1 == 32 || C1 == 64, "chunk 1 width");
  static_assert(D % 16 == 0 && D <= 128, "head_dim");
  static_assert(STAGES >= 2, "shared memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(Q1_OFF % 1024 == 0 && K1_OFF % 1024 == 0 && V1_OFF % 1024 == 0 && KV_BYTES % 1024 == 0 &&
                    Q_BYTES % 1024 == 0,
                "1024-byte alignment of swizzled tiles");
};

// One work item: query tiles 2 qp and 2 qp + 1 of head h of image b.
struct AttnItem {
  int qp, h, b, N, tok0, nkv, bh;
};

// Decodes item `it` (query-tile pair fastest, then head, then image, so that items
// running at the same time share K and V through L2).  False when the pair lies past
// the end of a smaller image of a packed batch: that item has no work.
template <int BM, int BN>
__device__ __forceinline__ bool attn_item(const AttnParams& p, int nqp, int it, AttnItem& w) {
  w.qp = it % nqp;
  const int rest = it / nqp;
  w.h = rest % p.H;
  w.b = rest / p.H;
  w.N = p.varlen ? p.vl.tok_off[w.b + 1] - p.vl.tok_off[w.b] : p.N;
  w.tok0 = p.varlen ? p.vl.tok_off[w.b] : w.b * p.N;
  w.nkv = (w.N + BN - 1) / BN;
  w.bh = w.b * p.H + w.h;
  return w.qp * 2 * BM < w.N;
}

// The CTA's work units.  Its first units are whole items (both query tiles), taken
// with a stride of the grid over the first sched_full items; the items left after the
// last full round form a tail of one unit per CTA, in which sched_tail_split items are
// cut into two single-tile units (tmask 1 or 2), so that the tail spreads over more SMs
// (a CTA with one query tile finishes its unit sooner: its softmax does not share the
// SM).  k-th unit of this CTA: 0 none left, 1 a unit, 2 an empty unit (an item past the
// end of a smaller image of a packed batch).
template <int BM, int BN>
__device__ __forceinline__ int attn_unit(const AttnParams& p, int nqp, int k, AttnItem& w, int& tmask) {
  const int c = blockIdx.x;
  int it = c + k * static_cast<int>(gridDim.x);
  tmask = 3;
  if (it >= p.sched_full) {
    const int kt = (p.sched_full - c + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
    const int s = p.sched_tail_split;
    if (k != kt || c >= p.sched_tail_pairs + s) return 0;
    if (c < 2 * s) {
      it = p.sched_full + (c >> 1);
      tmask = 1 << (c & 1);
    } else {
      it = p.sched_full + s + (c - 2 * s);
    }
  }
  return attn_item<BM, BN>(p, nqp, it, w) ? 1 : 2;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > VT_WAIT_LIMIT_NS) {
      atomicOr(&g_attn_err, VT_DEVERR_TIMEOUT);
      return;
    }
  }
}

template <int D>
__device__ __forceinline__ uint64_t qk_desc(uint32_t tile_addr, int ks) {
  using S = AttnShape<D>;
  const int c = ks * 16;
  if (c < S::C0) return smem_desc(tile_addr + c * 2, S::SBO0, S::LAY0);
  return smem_desc(tile_addr + S::BM * S::C0 * 2 + (c - S::C0) * 2, S::SBO1, S::LAY1);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tcgen05(const __grid_constant__ CUtensorMap tmQ0, const __grid_constant__ CUtensorMap tmQ1,
                     const __grid_constant__ CUtensorMap tmK0, const __grid_constant__ CUtensorMap tmK1,
                     const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using S = AttnShape<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                               // two query tiles
  uint8_t* sKV = sQ + 2 * S::Q_BYTES;               // per stage: K tile then V^T tile
  uint8_t* sP = sKV + S::STAGES * S::KV_BYTES;      // one P tile per query tile
  uint64_t* bar = reinterpret_cast<uint64_t*>(sP + 2 * S::P_BYTES);
  uint64_t* q_full = bar;
  uint64_t* kv_full = bar + 1;
  uint64_t* kv_empty = kv_full + S::STAGES;
  uint64_t* s_full = kv_empty + S::STAGES;  // [2], per query tile
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 2;
  uint64_t* q_empty = drain + 1;  // the last score products of an item have read Q
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* armed = const_cast<int*>(abort_flag + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nqp = (p.N + 2 * S::BM - 1) / (2 * S::BM);  // query-tile pairs of the longest image

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      armed[s] = -1;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(q_empty, 1);
    armed[S::STAGES] = -1;  // query tiles
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(&g_attn_err) != 0) ? 1 : 0;
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
      // -------------------------------------------------------------- loads
      tma_prefetch_desc(&tmQ0);
      tma_prefetch_desc(&tmK0);
      tma_prefetch_desc(&tmV);
      uint32_t G = 0, I = 0;  // key-tile steps and units loaded so far by this CTA
      bool ok = true;
      for (int k = 0; ok; ++k) {
        AttnItem w;
        int tmask;
        const int ru = attn_unit<S::BM, S::BN>(p, nqp, k, w, tmask);
        if (ru == 0) break;
        if (ru == 2) continue;
        // Q is single-buffered: the previous unit's score products must have read it.
        if (I > 0 && !mbar_wait(q_empty, (I - 1) & 1, abort_flag, &g_attn_err)) break;
        const int qrow = w.tok0 * p.H + w.h * w.N + w.qp * 2 * S::BM;
        mbar_arrive_expect_tx(q_full, (tmask == 3 ? 2 : 1) * S::Q_BYTES);
        for (int t = 0; t < 2; ++t) {
          if (!((tmask >> t) & 1)) continue;
          tma_load_2d(sQ + t * S::Q_BYTES, &tmQ0, q_full, 0, qrow + t * S::BM);
          if (S::C1) tma_load_2d(sQ + t * S::Q_BYTES + S::Q1_OFF, &tmQ1, q_full, S::C0, qrow + t * S::BM);
        }
        armed[S::STAGES] = static_cast<int>(I & 1);
        ++I;
        const int krow = w.tok0 * p.H + w.h * w.N;
        const int vrow = w.bh * D;
        for (int j = 0; j < w.nkv; ++j, ++G) {
          const int s = G % S::STAGES;
          const uint32_t ph = (G / S::STAGES) & 1;
          if (!mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, &g_attn_err)) {
            ok = false;
            break;
          }
          uint8_t* sK = sKV + s * S::KV_BYTES;
          uint8_t* sV = sK + S::K_BYTES;
          mbar_arrive_expect_tx(&kv_full[s], S::KV_BYTES);
          tma_load_2d(sK, &tmK0, &kv_full[s], 0, krow + j * S::BN);
          if (S::C1) tma_load_2d(sK + S::K1_OFF, &tmK1, &kv_full[s], S::C0, krow + j * S::BN);
          tma_load_2d(sV, &tmV, &kv_full[s], j * S::BN, vrow);
          tma_load_2d(sV + S::V1_OFF, &tmV, &kv_full[s], j * S::BN + 64, vrow);
          armed[s] = static_cast<int>(ph);
        }
      }
      if (*abort_flag) {
        if (armed[S::STAGES] >= 0) drain_wait(q_full, static_cast<uint32_t>(armed[S::STAGES]));
        for (int s = 0; s < S::STAGES; ++s)
          if (armed[s] >= 0) drain_wait(&kv_full[s], static_cast<uint32_t>(armed[s]));
      }
    }
  } else if (!skip && warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, S::BN);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D);
      bool issued = false, ok = true;
      // O_t += P_t V for query tile t and the key tile of step g (j-th of its unit); c:
      // the number of earlier steps in which tile t took part (its barrier phases).
      auto issue_pv = [&](int t, uint32_t g, uint32_t c, int j) -> bool {
        if (!mbar_wait(&p_full[t], c & 1, abort_flag, &g_attn_err)) return false;
        tc_fence_after();
        const uint32_t p_addr = smem_u32(sP + t * S::P_BYTES);
        const uint32_t v_addr = smem_u32(sKV + (g % S::STAGES) * S::KV_BYTES + S::K_BYTES);
        const uint32_t tO = tmem + t * 256 + 128;
#pragma unroll
        for (int ks = 0; ks < S::BN / 16; ++ks) {
          const uint64_t ad = smem_desc(p_addr + (ks >> 2) * (S::BM * 128) + (ks & 3) * 32, 1024, 2);
          const uint64_t bd = smem_desc(v_addr + (ks >> 2) * S::V1_OFF + (ks & 3) * 32, 1024, 2);
          umma_bf16(tO, ad, bd, idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&o_done[t]);
        return true;
      };
      // The P V products of step g are issued after the score products of step g + 1,
      // which may belong to the next unit: the tensor pipe works on those while the
      // softmax warps finish step g.  pend_j < 0: nothing pending.
      int pend_j = -1, pend_mask = 0;
      uint32_t pend_g = 0, pend_c[2] = {0, 0};
      uint32_t G = 0, I = 0;
      uint32_t C[2] = {0, 0};  // steps in which query tile t took part
      auto flush = [&]() -> bool {
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (((pend_mask >> t) & 1) && !issue_pv(t, pend_g, pend_c[t], pend_j)) return false;
        umma_commit(&kv_empty[pend_g % S::STAGES]);
        return true;
      };
      for (int k = 0; ok; ++k) {
        AttnItem w;
        int tmask;
        const int ru = attn_unit<S::BM, S::BN>(p, nqp, k, w, tmask);
        if (ru == 0) break;
        if (ru == 2) continue;
        // Unit boundary: the previous unit's last P V products go first unless this unit's
        // query tiles have already arrived (then its first score products run while the
        // softmax finishes the last step).
        if (pend_j >= 0 && !mbar_test(q_full, I & 1)) {
          if (!(ok = flush())) break;
          pend_j = -1;
        }
        if (!mbar_wait(q_full, I & 1, abort_flag, &g_attn_err)) {
          ok = false;
          break;
        }
        ++I;
        for (int j = 0; j < w.nkv; ++j, ++G) {
          const int s = G % S::STAGES;
          if (!mbar_wait(&kv_full[s], (G / S::STAGES) & 1, abort_flag, &g_attn_err)) {
            ok = false;
            break;
          }
          const uint32_t k_addr = smem_u32(sKV + s * S::KV_BYTES);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!ok || !((tmask >> t) & 1)) continue;
            // S_t is single-buffered: the softmax must have read S_t of tile t's last step.
            if (C[t] >= 1 && !mbar_wait(&s_free[t], (C[t] - 1) & 1, abort_flag, &g_attn_err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(sQ + t * S::Q_BYTES);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              umma_bf16(tmem + t * 256, qk_desc<D>(q_addr, ks), qk_desc<D>(k_addr, ks), idesc_s, ks > 0 ? 1u : 0u);
            issued = true;
            umma_commit(&s_full[t]);
            ++C[t];
          }
          if (!ok) break;
          if (j == w.nkv - 1) umma_commit(q_empty);
          if (pend_j >= 0 && !(ok = flush())) break;
          pend_j = j;
          pend_g = G;
          pend_mask = tmask;
          pend_c[0] = C[0] - 1;
          pend_c[1] = C[1] - 1;
        }
      }
      if (ok && pend_j >= 0) ok = flush();
      if (*abort_flag && issued) {
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (!skip) {
    // ------------------------------------------------------------- softmax
    const int t = (warp - 2) >> 2;   // query tile of this warpgroup
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + t * 256 + lane_off;
    const uint32_t tO = tS + 128;
    const float sl2 = p.scale * 1.4426950408889634f;  // scale * log2(e)
    uint8_t* pbuf = sP + t * S::P_BYTES;
    bool ok = true;
    uint32_t G = 0;  // steps in which this warpgroup's query tile took part
    for (int k = 0; ok; ++k) {
      int Nw, nkv;
      {
        AttnItem w;
        int tmask;
        const int ru = attn_unit<S::BM, S::BN>(p, nqp, k, w, tmask);
        if (ru == 0) break;
        if (ru == 2 || !((tmask >> t) & 1)) continue;
        Nw = w.N;
        nkv = w.nkv;
      }
      float m_ref = -INFINITY;  // running maximum of s * sl2 used as the exponent origin
      float l = 0.f;
      for (int j = 0; j < nkv; ++j, ++G) {
        if (!mbar_wait(&s_full[t], G & 1, abort_flag, &g_attn_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[S::BN];
        {
          uint32_t raw[S::BN];
          tmem_ld128(tS, raw);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < S::BN; ++c) s[c] = __uint_as_float(raw[c]);
        }
        tc_fence_before();
        mbar_arrive(&s_free[t]);
        const int valid = Nw - j * S::BN;
        if (valid < S::BN) {
#pragma unroll
          for (int c = 0; c < S::BN; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        // Row maximum: four independent chains of three-input maxima.
        float a4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c + 8 <= S::BN; c += 8)
#pragma unroll
          for (int i = 0; i < 4; ++i) a4[i] = fmax3(a4[i], s[c + i], s[c + 4 + i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) a4[i] = fmaxf(a4[i], s[S::BN - 4 + i]);
        const float mx = fmax3(a4[0], a4[1], fmaxf(a4[2], a4[3]));
        const float m_new = mx * sl2;
        bool need = false;
        if (j == 0) {
          m_ref = m_new;
        } else {
          need = m_new > m_ref + 8.0f;
          // P_t V of the previous step must be complete before P_t is overwritten and
          // before O_t is rescaled (at j = 0 the previous item's output wait did this).
          if (!mbar_wait(&o_done[t], (G - 1) & 1, abort_flag, &g_attn_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const bool any_need = __any_sync(0xffffffffu, need);
        const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
        if (need) {
          m_ref = m_new;
          l *= alpha;
        }
        // P = exp2(s * sl2 - m_ref), written bf16 in the 128-byte-swizzled K-major layout.
        const float2 sl2x2 = make_float2(sl2, sl2), negx2 = make_float2(-m_ref, -m_ref);
        float2 l4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c16 = 0; c16 < S::BN / 8; ++c16) {
          float e[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 x = ffma2(make_float2(s[c16 * 8 + 2 * q], s[c16 * 8 + 2 * q + 1]), sl2x2, negx2);
            const float2 y = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            e[2 * q] = y.x;
            e[2 * q + 1] = y.y;
            l4[q] = fadd2(l4[q], y);
          }
          const int blk = c16 >> 3, cc = c16 & 7;
          uint4* dst = reinterpret_cast<uint4*>(pbuf + blk * (S::BM * 128) + r * 128 + ((cc ^ (r & 7)) << 4));
          *dst = pack_bf16x8(e);
        }
        const float2 l2 = fadd2(fadd2(l4[0], l4[1]), fadd2(l4[2], l4[3]));
        l += l2.x + l2.y;
        if (any_need) {
          // Scale O_t to the new exponent origin before P_t V_j accumulates into it (the
          // wait on P_t V_{j-1} above made O_t stable).
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            uint32_t o[16];
            tmem_ld16(tO + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(tO + c, o);
          }
          tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // The last P V product of the item; its completion also frees P_t and O_t for
      // the next item.
      if (!(ok = mbar_wait(&o_done[t], (G - 1) & 1, abort_flag, &g_attn_err))) break;
      tc_fence_after();
      float o[D];
      load_cols<D>(tO, o);
      AttnItem w;  // decoded again rather than kept live through the step loop
      int tmask;
      attn_unit<S::BM, S::BN>(p, nqp, k, w, tmask);
      const int n = (w.qp * 2 + t) * S::BM + r;
      if (p.lse && n < w.N) p.lse[static_cast<size_t>(w.bh) * p.ld_lse + n] = m_ref + __log2f(l);
      if (n < w.N) {
        const float inv = 1.0f / l;
#pragma unroll
        for (int i = 0; i < D; ++i) o[i] *= inv;
        bf16* dst = static_cast<bf16*>(p.o) + (static_cast<size_t>(w.tok0) + n) * (p.H * D) + w.h * D;
#pragma unroll
        for (int g = 0; g < D / 8; ++g) reinterpret_cast<uint4*>(dst)[g] = pack_bf16x8(o + 8 * g);
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

template <int D>
cudaError_t launch_d(const AttnParams& p, cudaStream_t stream) {
  using S = AttnShape<D>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_fwd_tcgen05<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const uint64_t rows = static_cast<uint64_t>(p.varlen ? p.vl.tok_off[p.vl.count] : p.B * p.N) * p.H;
  CUtensorMap q0, q1, k0, k1, v;
  if (!make_tmap_2d(&q0, p.q, rows, D, D, S::BM, S::C0, S::SW0)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&k0, p.k, rows, D, D, S::BN, S::C0, S::SW0)) return cudaErrorInvalidValue;
  if (S::C1) {
    if (!make_tmap_2d(&q1, p.q, rows, D, D, S::BM, S::C1, S::SW1)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&k1, p.k, rows, D, D, S::BN, S::C1, S::SW1)) return cudaErrorInvalidValue;
  } else {
    q1 = q0;
    k1 = k0;
  }
  if (!make_tmap_2d(&v, p.vt, static_cast<uint64_t>(p.B) * p.H * D, p.varlen ? p.ld_vt : p.N, p.ld_vt, D, 64, 128))
    return cudaErrorInvalidValue;
  // Persistent: one CTA per SM (shared memory and the 512 TMEM columns allow no more).
  // Full rounds of whole items, then a tail in which as many of the remaining items as
  // there are otherwise idle SMs are cut into single-tile units.  Packed batches of
  // mixed sizes (which have empty items) run whole items only.
  AttnParams ps = p;
  const long items = static_cast<long>((p.N + 2 * S::BM - 1) / (2 * S::BM)) * p.H * p.B;
  const int sms = device_sm_count();
  int grid;
  if (p.varlen) {
    ps.sched_full = static_cast<int>(items);
    ps.sched_tail_pairs = ps.sched_tail_split = 0;
    grid = static_cast<int>(items < sms ? items : sms);
  } else {
    const long full = items / sms * sms, rest = items - full;
    const long split = rest < sms - rest ? rest : sms - rest;
    ps.sched_full = static_cast<int>(full);
    ps.sched_tail_pairs = static_cast<int>(rest);
    ps.sched_tail_split = static_cast<int>(split);
    grid = full > 0 ? sms : static_cast<int>(rest + split);
  }
  if (grid <= 0) return cudaSuccess;
  attn_fwd_tcgen05<D><<<grid, kThreads, S::SMEM_BYTES, stream>>>(q0, q1, k0, k1, v, ps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnParams& p, cudaStream_t stream) {
  if (p.B <= 0 || p.H <= 0 || p.N <= 0) return cudaSuccess;
  switch (p.D) {
    case 32: return launch_d<32>(p, stream);
    case 64: return launch_d<64>(p, stream);
    case 80: return launch_d<80>(p, stream);
    case 96: return launch_d<96>(p, stream);
    default: return cudaErrorNotSupported;
  }
}

unsigned int attention_read_clear_error(cudaStream_t stream) {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_attn_err, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return 0;
  cudaStreamSynchronize(stream);
  if (v) {
    cudaMemcpyToSymbolAsync(g_attn_err, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    cudaStreamSynchronize(stream);
  }
  return v;
}

}  // namespace vt
