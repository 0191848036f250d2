// Persistent bf16 GEMM for sm_100a: TMA -> shared-memory ring -> tcgen05.mma (fp32
// accumulator in TMEM) -> tcgen05.ld epilogue with fused bias / GELU / residual, or
// with the QKV epilogue that applies 3D RoPE and writes the attention layouts.
//
// Computes out[M, N] = act(A[M, K] * W[N, K]^T + bias) (+ resid), the form of every
// linear layer of the tower and projector ("MiniMax-M3 Vision" model card,
// Architecture table: Conv3d patch embed, qkv / o projections, MLP 1280 -> 5120 -> 1280
// with GELU, projector Linear(1280,6144), GELU, Linear(6144,6144), Linear(24576,6144),
// GELU, Linear(6144,6144)).
//
// Two kernels share one epilogue:
//  * gemm_bf16_tcgen05: one CTA per 128 x BN tile.
//  * gemm_bf16_tcgen05_pair: a cluster of two CTAs (the two SMs of a TPC) per
//    256 x BN tile with tcgen05.mma.cta_group::2.  Each CTA stages its own 128 rows of A
//    and BN/2 rows of B, so an SM streams 32 KB of operands per 64-deep K step instead
//    of 48 KB, and six stages fit in shared memory.  The even CTA issues the MMAs and
//    both CTAs drain their own 128 accumulator rows.  No load uses multicast.
// CTA = 6 or 10 warps: warp 0 issues TMA loads, warp 1 allocates TMEM and issues the MMAs
// (one thread), the rest run the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).  The
// plain epilogue (bias / GELU / residual) has two groups of four warps that take the
// 32-column chunks of a tile alternately, so two warps per SM sub-partition hide each
// other's load and store latency (short-K GEMMs are otherwise bound by their epilogue);
// the QKV epilogue, which keeps a whole head per thread, has one group.
// K steps are 64 deep (one 128-byte swizzle atom); two TMEM accumulators let the
// epilogue of one tile overlap the main loop of the next.  Tiles are walked m-fastest
// by a persistent grid, so concurrently running CTAs share each weight tile via L2.
#include "internal.h"
#include "ptx.cuh"

namespace vt {
namespace {

__device__ unsigned int g_gemm_err;

constexpr int kBM = 128;
constexpr int kBK = 64;
// Epilogue warp groups and threads per CTA for an epilogue kind.
template <class RL>
struct Epi {
  static constexpr int GROUPS = RL::D == 0 ? 2 : 1;
  static constexpr int THREADS = 64 + 128 * GROUPS;
};

template <int BN, bool PAIR>
struct GemmShape {
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // rows of B this CTA stages
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = B_ROWS * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = BN <= 128 ? 128 : 256;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = 256;
  // Output staging of the plain epilogue: per epilogue warp two [32 x 32] bf16 boxes.
  static constexpr int EPI_BOX = 32 * 32 * 2;
  static constexpr int EPI_BYTES = 8 * 2 * EPI_BOX;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "tiles must keep 1024-byte alignment");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N");
  static_assert(!PAIR || (BN / 2) % 8 == 0, "half of B must be whole 8-row groups");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Head layouts the QKV epilogue supports: head_dim and the three RoPE sections.
struct Rope0 { static constexpr int D = 0, S0 = 0, S1 = 0, S2 = 0; };
struct Rope80 { static constexpr int D = 80, S0 = 16, S1 = 32, S2 = 32; };
struct Rope32 { static constexpr int D = 32, S0 = 8, S1 = 12, S2 = 12; };

// Rotates the pairs (off + j, off + j + S/2) of one axis block in place.
template <int OFF, int S>
__device__ __forceinline__ void rope_block(float* v, const float2* tab_axis_pos) {
#pragma unroll
  for (int j = 0; j < S / 2; ++j) {
    const float2 cs = tab_axis_pos[j];
    const float a = v[OFF + j], b = v[OFF + j + S / 2];
    v[OFF + j] = a * cs.x - b * cs.y;
    v[OFF + j + S / 2] = b * cs.x + a * cs.y;
  }
}

// Bounded wait used only while tearing down after an abort.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > VT_WAIT_LIMIT_NS) {
      atomicOr(&g_gemm_err, VT_DEVERR_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = global_ns();
  while (global_ns() - t0 < ns) {
  }
}

// Bulk tensor store of a [32 x 32] box from this CTA's shared memory (the caller's
// async-proxy fence precedes it), tracked by the issuing thread's bulk async-groups.
__device__ __forceinline__ void tma_store_2d(const void* map, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most one committed group still reads its shared-memory source.
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Row and column tile of output tile `tile` in the order p.n_fastest selects.
__host__ __device__ __forceinline__ int tile_row(const GemmParams& p, int tile, int m_tiles, int n_tiles) {
  return p.n_fastest ? tile / n_tiles : tile % m_tiles;
}
__host__ __device__ __forceinline__ int tile_col(const GemmParams& p, int tile, int m_tiles, int n_tiles) {
  return p.n_fastest ? tile % n_tiles : tile / m_tiles;
}

// Work item i (0, 1, ...) of CTA pair `pair` of P: output tile `tile` over K steps
// [kb0, kb1).  Whole tiles come in rounds of P; with a split-K tail (p.sk_part) the
// tiles from p.sk_full on are cut into p.sk_split K ranges each, and pair u takes range
// u % sk_split of tile sk_full + u / sk_split as its last item (unit = u; -1 for a whole
// tile).  Every role of the kernel walks the same items.
__device__ __forceinline__ bool pair_work(const GemmParams& p, int pair, int P, int T, int nk, int i, int& tile,
                                          int& kb0, int& kb1, int& unit) {
  const int F = p.sk_part ? p.sk_full : T;
  const int whole = pair < F ? (F - pair + P - 1) / P : 0;
  if (i < whole) {
    tile = pair + i * P;
    kb0 = 0;
    kb1 = nk;
    unit = -1;
    return true;
  }
  if (!p.sk_part || i != whole || pair >= (T - F) * p.sk_split) return false;
  const int sp = pair % p.sk_split;
  tile = F + pair / p.sk_split;
  kb0 = sp * nk / p.sk_split;
  kb1 = (sp + 1) * nk / p.sk_split;
  unit = pair;
  return true;
}

// Drains one accumulator: this thread's row `row`, columns [col0, col0 + BN), the
// warp's TMEM lane quadrant at t_row.  Waits for the accumulator (tfull, phase
// `parity`) itself, after issuing the loads it can issue early.  Returns false on abort.
// Group `grp` of Epi<RL>::GROUPS drains 32-column chunks grp, grp + GROUPS, ... (plain
// epilogue); the QKV epilogue has one group.
//
// The plain epilogue writes `out` through shared memory: each warp packs its 32 rows x 32
// columns into one of its two 64-byte-swizzled staging boxes (`stage`, alternating with
// `sbuf`) and one lane stores the box with a bulk tensor store (tmC: [M, N] with row
// stride ldo, box 32 x 32), which clips rows and columns past the matrix.
template <int BN, class RL, bool PAIR>
__device__ __forceinline__ bool epilogue_tile(const GemmParams& p, int row, int col0, uint32_t t_row, uint64_t* tfull,
                                              uint32_t parity, volatile int* abort_flag, int grp,
                                              const CUtensorMap* tmC, const CUtensorMap* tmZ, uint8_t* stage,
                                              int& sbuf) {
  auto wait_acc = [&]() -> bool {
    const bool ok = PAIR ? mbar_wait_cluster(tfull, parity, abort_flag, &g_gemm_err)
                         : mbar_wait(tfull, parity, abort_flag, &g_gemm_err);
    if (ok) tc_fence_after();
    return ok;
  };
  if constexpr (RL::D == 0) {
    const bf16* bias = static_cast<const bf16*>(p.bias);
    const bf16* resid = static_cast<const bf16*>(p.resid);
    // Bias and residual of a 32-column chunk are loaded one chunk ahead (the first
    // chunk before waiting for the accumulator) so that no global-load latency sits
    // between the TMEM read and the store.
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    auto prefetch = [&](int col, uint4* bq, uint4* rq) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int cg = col + 8 * g;
        bq[g] = (bias && cg < p.N) ? __ldg(reinterpret_cast<const uint4*>(bias + cg)) : zero;
        rq[g] = (resid && cg < p.N && row < p.M)
                    ? *reinterpret_cast<const uint4*>(resid + static_cast<size_t>(row) * p.ldr + cg)
                    : zero;
      }
    };
    constexpr int STEP = 32 * Epi<RL>::GROUPS;
    uint4 bq[4], rq[4];
    prefetch(col0 + 32 * grp, bq, rq);
    if (!wait_acc()) return false;
#pragma unroll 1
    for (int c0 = 32 * grp; c0 < BN; c0 += STEP) {
      const int col = col0 + c0;
      if (col >= p.N) break;
      uint4 bn_[4] = {zero, zero, zero, zero}, rn_[4] = {zero, zero, zero, zero};
      if (c0 + STEP < BN) prefetch(col + STEP, bn_, rn_);
      float v[32];
      load_cols<32>(t_row + c0, v);
      const int lane = threadIdx.x & 31;
      // Stages the warp's 32 x 32 box of `vals` (row = lane; 16-byte chunk g of a 64-byte
      // row at g ^ ((lane >> 1) & 3), the 64-byte swizzle) and stores it with one bulk copy.
      auto store_box = [&](const CUtensorMap* map, const float* vals) {
        uint8_t* box = stage + sbuf * (32 * 32 * 2);
        if (lane == 0) bulk_wait_read1();  // the store that last read this box is done
        __syncwarp();
#pragma unroll
        for (int g = 0; g < 4; ++g)
          *reinterpret_cast<uint4*>(box + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) = pack_bf16x8(vals + 8 * g);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(map, box, col, row - lane);
          bulk_commit();
        }
        sbuf ^= 1;
      };
      if (bias) {
#pragma unroll
        for (int g = 0; g < 4; ++g)
          if (col + 8 * g < p.N) add_bf16x8(v + 8 * g, bq[g]);
      }
      if (p.pre_out) store_box(tmZ, v);  // pre-activation kept for a later backward
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int cg = col + 8 * g;
        if (cg < p.N) {
          if (p.act >= ACT_DGELU_TANH) {
            // backward of GELU: scale by gelu'(pre-activation), which `resid` carries
            const uint32_t w[4] = {rq[g].x, rq[g].y, rq[g].z, rq[g].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 z = unpack_bf16x2(w[i]);
              const bool th = p.act == ACT_DGELU_TANH;
              v[8 * g + 2 * i] *= th ? gelu_tanh_grad(z.x) : gelu_erf_grad(z.x);
              v[8 * g + 2 * i + 1] *= th ? gelu_tanh_grad(z.y) : gelu_erf_grad(z.y);
            }
          } else if (p.act == ACT_GELU_TANH) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 y = gelu_tanh2(make_float2(v[8 * g + 2 * i], v[8 * g + 2 * i + 1]));
              v[8 * g + 2 * i] = y.x;
              v[8 * g + 2 * i + 1] = y.y;
            }
          } else if (p.act == ACT_GELU_ERF) {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[8 * g + i] = gelu_erf(v[8 * g + i]);
          }
          if (resid && p.act < ACT_DGELU_TANH) add_bf16x8(v + 8 * g, rq[g]);
        }
      }
      store_box(tmC, v);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        bq[g] = bn_[g];
        rq[g] = rn_[g];
      }
    }
  } else {
    if (!wait_acc()) return false;
    constexpr int D = RL::D;
    constexpr int HPT = BN / D;
    const bf16* bias = static_cast<const bf16*>(p.bias);
    const int width = p.heads * D;
    // Token n of image b, whose tokens start at packed row tok0 and number ntok.
    int n = 0, tp = 0, hp = 0, wp = 0, ntok = p.ntok, ld_vt = p.ld_vt;
    size_t tok0 = 0, vt0 = 0;
    if (row < p.M) {
      if (p.varlen) {
        const int b = varlen_image(p.vl, row);
        tok0 = static_cast<size_t>(p.vl.tok_off[b]);
        ntok = p.vl.tok_off[b + 1] - p.vl.tok_off[b];
        n = row - p.vl.tok_off[b];
        ld_vt = p.vl.ld_vt[b];
        vt0 = static_cast<size_t>(p.vl.vt_off[b]);
        token_position(n, p.vl.gh[b], p.vl.gw[b], p.order, &tp, &hp, &wp);
      } else {
        const int b = row / p.ntok;
        n = row - b * p.ntok;
        tok0 = static_cast<size_t>(b) * p.ntok;
        vt0 = static_cast<size_t>(b) * p.heads * D * p.ld_vt;
        token_position(n, p.gh, p.gw, p.order, &tp, &hp, &wp);
      }
    }
#pragma unroll 1
    for (int hh = 0; hh < HPT; ++hh) {
      const int col = col0 + hh * D;
      if (col >= p.N) break;
      float v[D];
      load_cols<D>(t_row + hh * D, v);
      if (bias) {
#pragma unroll
        for (int g = 0; g < D / 8; ++g) add_bf16x8(v + 8 * g, *reinterpret_cast<const uint4*>(bias + col + 8 * g));
      }
      const int which = col / width;
      const int head = (col - which * width) / D;
      if (row < p.M) {
        if (which < 2) {
          if (p.rope) {
            const float2* tab = p.rope_tab;
            rope_block<0, RL::S0>(v, tab + (static_cast<size_t>(0 * kRopeMaxPos + tp) * kRopePairs));
            rope_block<RL::S0, RL::S1>(v, tab + (static_cast<size_t>(1 * kRopeMaxPos + hp) * kRopePairs));
            rope_block<RL::S0 + RL::S1, RL::S2>(v, tab + (static_cast<size_t>(2 * kRopeMaxPos + wp) * kRopePairs));
          }
          // [heads, ntok, D] block of this image, which starts at token tok0
          bf16* dst = static_cast<bf16*>(which == 0 ? p.q : p.k) +
                      (tok0 * p.heads + static_cast<size_t>(head) * ntok + n) * D;
#pragma unroll
          for (int g = 0; g < D / 8; ++g) reinterpret_cast<uint4*>(dst)[g] = pack_bf16x8(v + 8 * g);
        } else {
          // [heads, D, ld_vt] block of this image at vt0
          bf16* dst = static_cast<bf16*>(p.vt) + vt0 + static_cast<size_t>(head) * D * ld_vt + n;
#pragma unroll
          for (int d = 0; d < D; ++d) dst[static_cast<size_t>(d) * ld_vt] = __float2bfloat16_rn(v[d]);
        }
      }
    }
  }
  return true;
}

// ------------------------------------------------------------ one CTA per tile

template <int BN, class RL>
__global__ void __launch_bounds__(Epi<RL>::THREADS, 1)
    gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmZ,
                      const GemmParams p) {
  using S = GemmShape<BN, false>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::STAGES * S::A_BYTES;
  uint8_t* sEpi = sB + S::STAGES * S::B_BYTES;  // output staging, two boxes per epilogue warp
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + S::EPI_BYTES);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* armed = const_cast<int*>(abort_flag + 1);  // last phase armed per stage, -1 = never

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (p.M + kBM - 1) / kBM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int nk = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      armed[s] = -1;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128 * Epi<RL>::GROUPS);
    }
    mbar_init(drain, 1);
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(&g_gemm_err) != 0) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool skip = *abort_flag != 0;

  if (!skip && warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int mb = tile_row(p, tile, m_tiles, n_tiles), nb = tile_col(p, tile, m_tiles, n_tiles);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, &g_gemm_err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
          tma_load_2d(sA + stage * S::A_BYTES, &tmA, &full[stage], kb * kBK, mb * kBM);
          tma_load_2d(sB + stage * S::B_BYTES, &tmB, &full[stage], kb * kBK, nb * BN);
          armed[stage] = static_cast<int>(phase);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {  // let every load already issued land before the CTA exits
        for (int s = 0; s < S::STAGES; ++s)
          if (armed[s] >= 0) drain_wait(&full[s], static_cast<uint32_t>(armed[s]));
      } else {
        // Wait until the MMAs released every stage (their commits arrive asynchronously).
        for (int i = 0; i < S::STAGES; ++i) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, &g_gemm_err)) break;
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (!skip && warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
      // Descriptors of stage 0, computed once: later stages and K steps add to the
      // start-address field (address / 16; shared addresses stay below 256 KB).
      const uint64_t a_desc0 = smem_desc(smem_u32(sA), 1024, 2), b_desc0 = smem_desc(smem_u32(sB), 1024, 2);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&tempty[acc], ((it >> 1) & 1) ^ 1u, abort_flag, &g_gemm_err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * S::ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, &g_gemm_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(stage * (S::A_BYTES >> 4));
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(stage * (S::B_BYTES >> 4));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      if (*abort_flag && issued_any) {  // wait for MMAs in flight before TMEM is freed
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (!skip) {
    // ------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    uint8_t* stage = sEpi + (warp - 2) * 2 * S::EPI_BOX;
    int sbuf = 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const int mb = tile_row(p, tile, m_tiles, n_tiles), nb = tile_col(p, tile, m_tiles, n_tiles);
      const int row = mb * kBM + quad * 32 + lane;
      const uint32_t t_row = tmem_base + acc * S::ACC_COLS + (static_cast<uint32_t>(quad * 32) << 16);
      if (!epilogue_tile<BN, RL, false>(p, row, nb * BN, t_row, &tfull[acc], (it >> 1) & 1, abort_flag, grp, &tmC,
                                        &tmZ, stage, sbuf))
        break;
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
    if ((threadIdx.x & 31) == 0) bulk_wait_all();  // every staged box has reached memory
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

// ---------------------------------------------------- two CTAs per 256-row tile

template <int BN, class RL>
__global__ void __launch_bounds__(Epi<RL>::THREADS, 1)
    gemm_bf16_tcgen05_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmZ,
                           const GemmParams p) {
  using S = GemmShape<BN, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::STAGES * S::A_BYTES;
  uint8_t* sEpi = sB + S::STAGES * S::B_BYTES;  // output staging, two boxes per epilogue warp
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + S::EPI_BYTES);  // used in the even CTA
  uint64_t* empty = full + S::STAGES;                                          // both CTAs
  uint64_t* tfull = empty + S::STAGES;                                         // both CTAs
  uint64_t* tempty = tfull + 2;                                                // even CTA
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* armed = const_cast<int*>(abort_flag + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int m_tiles = (p.M + 2 * kBM - 1) / (2 * kBM);
  const int n_tiles = (p.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int nk = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      armed[s] = -1;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8 * Epi<RL>::GROUPS);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(&g_gemm_err) != 0) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // barrier inits and TMEM allocation visible to both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Both CTAs must take the same path: skip only if either saw an earlier error.
  const bool skip = *abort_flag != 0;

  if (!skip && warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // Both CTAs load their own halves; completion is counted on the even CTA's
      // full[stage], armed by the even CTA for the bytes of both.
      int stage = 0;
      uint32_t phase = 0;
      int tile, kb0, kb1, unit;
      for (int i = 0; pair_work(p, pair, num_pairs, num_tiles, nk, i, tile, kb0, kb1, unit); ++i) {
        const int mb = tile_row(p, tile, m_tiles, n_tiles), nb = tile_col(p, tile, m_tiles, n_tiles);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, abort_flag, &g_gemm_err)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * S::STAGE_BYTES);
          tma_load_2d_pair(sA + stage * S::A_BYTES, &tmA, full_leader, kb * kBK, mb * 2 * kBM + rank * kBM);
          tma_load_2d_pair(sB + stage * S::B_BYTES, &tmB, full_leader, kb * kBK, nb * BN + rank * (BN / 2));
          armed[stage] = static_cast<int>(phase);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        if (rank == 0)
          for (int s = 0; s < S::STAGES; ++s)
            if (armed[s] >= 0) drain_wait(&full[s], static_cast<uint32_t>(armed[s]));
      } else {
        // Wait until the MMAs released every stage, so that no arrival from the even
        // CTA's commits is still on its way to this CTA's barriers when it exits.
        for (int i = 0; i < S::STAGES; ++i) {
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, abort_flag, &g_gemm_err)) break;
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (!skip && warp == 1) {
    if (lane == 0 && rank == 0) {
      // -------------------------------------------------------- MMA (even CTA)
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, BN);
      // Descriptors of stage 0 and the cluster addresses of the stage-0 empty barriers,
      // computed once: the descriptor's start-address field holds address / 16 (shared
      // addresses stay below 256 KB, so adding stage and K-step offsets never carries out
      // of it), and the barriers of later stages follow at 8-byte steps.
      const uint64_t a_desc0 = smem_desc(smem_u32(sA), 1024, 2), b_desc0 = smem_desc(smem_u32(sB), 1024, 2);
      const uint32_t e_lead0 = mapa_shared(smem_u32(&empty[0]), 0), e_peer0 = mapa_shared(smem_u32(&empty[0]), 1);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool issued_any = false;
      int tile, kb0, kb1, unit;
      for (; pair_work(p, pair, num_pairs, num_tiles, nk, it, tile, kb0, kb1, unit); ++it) {
        const int acc = it & 1;
        if (!mbar_wait_cluster(&tempty[acc], ((it >> 1) & 1) ^ 1u, abort_flag, &g_gemm_err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * S::ACC_COLS;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_cluster(&full[stage], phase, abort_flag, &g_gemm_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(stage * (S::A_BYTES >> 4));
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(stage * (S::B_BYTES >> 4));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb > kb0 || kk != 0) ? 1u : 0u);
          issued_any = true;
          umma_commit_pair(e_lead0 + 8u * stage);
          umma_commit_pair(e_peer0 + 8u * stage);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        const uint32_t t_local = smem_u32(&tfull[acc]);
        umma_commit_pair(mapa_shared(t_local, 0));
        umma_commit_pair(mapa_shared(t_local, 1));
      }
      if (*abort_flag && issued_any) {
        umma_commit_pair(mapa_shared(smem_u32(drain), 0));
        drain_wait(drain, 0);
      }
    }
  } else if (!skip) {
    // ------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty[0]), 0), mapa_shared(smem_u32(&tempty[1]), 0)};
    uint8_t* stage = sEpi + (warp - 2) * 2 * S::EPI_BOX;
    int sbuf = 0;
    int it = 0;
    int tile, kb0, kb1, unit;
    for (; pair_work(p, pair, num_pairs, num_tiles, nk, it, tile, kb0, kb1, unit); ++it) {
      const int acc = it & 1;
      const int mb = tile_row(p, tile, m_tiles, n_tiles), nb = tile_col(p, tile, m_tiles, n_tiles);
      const int row = mb * 2 * kBM + rank * kBM + quad * 32 + lane;
      const uint32_t t_row = tmem_base + acc * S::ACC_COLS + (static_cast<uint32_t>(quad * 32) << 16);
      if (unit >= 0) {
        // A K range of a split tile: its fp32 partial sums go to scratch, row-major
        // [256][BN] per unit (each thread writes its row's 128 contiguous bytes per chunk),
        // so that the sum kernel reads and writes whole rows.
        if (!mbar_wait_cluster(&tfull[acc], (it >> 1) & 1, abort_flag, &g_gemm_err)) break;
        tc_fence_after();
        float* part = p.sk_part + (static_cast<size_t>(unit) * (2 * kBM) + rank * kBM + quad * 32 + lane) * BN;
#pragma unroll 1
        for (int c0 = 32 * grp; c0 < BN; c0 += 32 * Epi<RL>::GROUPS) {
          float v[32];
          load_cols<32>(t_row + c0, v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(part + c0)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      } else if (!epilogue_tile<BN, RL, true>(p, row, nb * BN, t_row, &tfull[acc], (it >> 1) & 1, abort_flag, grp,
                                              &tmC, &tmZ, stage, sbuf)) {
        break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
    }
    if (lane == 0) bulk_wait_all();  // every staged box has reached memory
  }

  // Neither CTA may leave while the pair's MMAs, loads or arrivals can still touch it.
  if (*abort_flag) spin_ns(20000);
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

// --------------------------------------------------------- split-K tail sum
constexpr int kMaxSplit = 8;  // K ranges per split tile at most

// out = epilogue(sum over s of part[tile's unit s]) for the split tiles of a pair
// product: the partials are added in unit order (the same order on every run), then
// bias, activation and residual as in epilogue_tile.  One thread per 4 consecutive
// columns of one row; a warp covers 128 contiguous columns, so its partial loads are
// 512 contiguous bytes and its residual loads and output stores 256.
template <int BN>
__global__ void __launch_bounds__(256) gemm_split_sum(const GemmParams p) {
  const int m_tiles = (p.M + 2 * kBM - 1) / (2 * kBM);
  constexpr int QUADS = BN / 4;  // four columns per thread: a warp covers 128 contiguous columns
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int g = static_cast<int>(i % QUADS);
  const long long rest = i / QUADS;
  const int r = static_cast<int>(rest % (2 * kBM));
  const int t = static_cast<int>(rest / (2 * kBM));  // split tile, 0-based after sk_full
  const int tile = p.sk_full + t;
  if (tile >= m_tiles * ((p.N + BN - 1) / BN)) return;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int row = tile_row(p, tile, m_tiles, n_tiles) * 2 * kBM + r;
  const int col = tile_col(p, tile, m_tiles, n_tiles) * BN + 4 * g;
  if (row >= p.M || col >= p.N) return;
  // every partial is loaded before the first add, so that the loads overlap
  float4 pv[kMaxSplit];
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) {
    if (s >= p.sk_split) break;
    pv[s] = *reinterpret_cast<const float4*>(p.sk_part + (static_cast<size_t>(t * p.sk_split + s) * (2 * kBM) + r) * BN +
                                             4 * g);
  }
  float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) {
    if (s >= p.sk_split) break;
    v[0] += pv[s].x;
    v[1] += pv[s].y;
    v[2] += pv[s].z;
    v[3] += pv[s].w;
  }
  auto add4 = [&](uint2 u) {
    const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
    v[0] += a.x;
    v[1] += a.y;
    v[2] += b.x;
    v[3] += b.y;
  };
  if (p.bias) add4(__ldg(reinterpret_cast<const uint2*>(static_cast<const bf16*>(p.bias) + col)));
  if (p.act == ACT_GELU_TANH) {  // the tile epilogue's packed form, so that split and whole tiles agree
#pragma unroll
    for (int c = 0; c < 4; c += 2) {
      const float2 y = gelu_tanh2(make_float2(v[c], v[c + 1]));
      v[c] = y.x;
      v[c + 1] = y.y;
    }
  } else if (p.act == ACT_GELU_ERF) {
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = gelu_erf(v[c]);
  }
  if (p.resid)
    add4(*reinterpret_cast<const uint2*>(static_cast<const bf16*>(p.resid) + static_cast<size_t>(row) * p.ldr + col));
  *reinterpret_cast<uint2*>(static_cast<bf16*>(p.out) + static_cast<size_t>(row) * p.ldo + col) =
      make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// ------------------------------------------------------------------- launch

// K ranges per tile for the split-K tail of a plain pair product, 1 for none.  Used when
// the tiles of the last round fill at most half of the pairs and K is long (at least 32
// steps: below that the tail sum costs about what the split saves, measured on B200 for
// the 1280-deep output projection), with at least eight K steps per range and an
// epilogue that the tail sum reproduces.
int split_factor(const GemmParams& p, int tiles, int pairs, int bn) {
  if (!p.sk_part || p.pre_out || p.act > ACT_GELU_ERF || p.N % 8) return 1;
  const int rem = tiles % pairs;
  if (rem == 0 || 2 * rem > pairs) return 1;
  const int nk = (p.K + kBK - 1) / kBK;
  if (nk < 32) return 1;
  int s = pairs / rem;
  if (s > nk / 8) s = nk / 8;
  if (s > kMaxSplit) s = kMaxSplit;
  if (static_cast<size_t>(rem) * s * 2 * kBM * bn * sizeof(float) > gemm_split_bytes()) return 1;
  return s > 1 ? s : 1;
}

template <int BN, class RL>
cudaError_t launch_one(const GemmParams& p, cudaStream_t stream) {
  using S = GemmShape<BN, false>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tcgen05<BN, RL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, p.A, p.M, p.K, p.lda, kBM, kBK, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, p.W, p.N, p.K, p.ldw, BN, kBK, 128)) return cudaErrorInvalidValue;
  CUtensorMap tc = tb, tz = tb;  // the QKV epilogue writes its own layouts
  if (RL::D == 0 && !make_tmap_2d(&tc, p.out, p.M, p.N, p.ldo, 32, 32, 64)) return cudaErrorInvalidValue;
  if (RL::D == 0 && p.pre_out && !make_tmap_2d(&tz, p.pre_out, p.M, p.N, p.ldo, 32, 32, 64))
    return cudaErrorInvalidValue;
  const int tiles = ((p.M + kBM - 1) / kBM) * ((p.N + BN - 1) / BN);
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  gemm_bf16_tcgen05<BN, RL><<<grid, Epi<RL>::THREADS, S::SMEM_BYTES, stream>>>(ta, tb, tc, tz, p);
  return cudaGetLastError();
}

template <int BN, class RL>
cudaError_t launch_pair(const GemmParams& p, cudaStream_t stream, int* kernels = nullptr) {
  using S = GemmShape<BN, true>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tcgen05_pair<BN, RL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, p.A, p.M, p.K, p.lda, kBM, kBK, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, p.W, p.N, p.K, p.ldw, BN / 2, kBK, 128)) return cudaErrorInvalidValue;
  CUtensorMap tc = tb, tz = tb;  // the QKV epilogue writes its own layouts
  if (RL::D == 0 && !make_tmap_2d(&tc, p.out, p.M, p.N, p.ldo, 32, 32, 64)) return cudaErrorInvalidValue;
  if (RL::D == 0 && p.pre_out && !make_tmap_2d(&tz, p.pre_out, p.M, p.N, p.ldo, 32, 32, 64))
    return cudaErrorInvalidValue;
  const int tiles = ((p.M + 2 * kBM - 1) / (2 * kBM)) * ((p.N + BN - 1) / BN);
  const int max_pairs = device_sm_count() / 2;
  int pairs = tiles < max_pairs ? tiles : max_pairs;
  GemmParams q = p;
  const int split = split_factor(p, tiles, max_pairs, BN);
  if (split > 1) {
    q.sk_full = tiles - tiles % max_pairs;
    q.sk_split = split;
    pairs = max_pairs;
  } else {
    q.sk_part = nullptr;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(Epi<RL>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_bf16_tcgen05_pair<BN, RL>, ta, tb, tc, tz, q);
  if (e != cudaSuccess) return e;
  if (kernels) *kernels = split > 1 ? 2 : 1;
  if (split > 1) {
    const long long threads = static_cast<long long>(tiles - q.sk_full) * (BN / 4) * (2 * kBM);
    gemm_split_sum<BN><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(q);
  }
  return cudaGetLastError();
}

}  // namespace

size_t gemm_split_bytes() { return static_cast<size_t>(device_sm_count() / 2) * 2 * kBM * 256 * sizeof(float); }

cudaError_t launch_gemm(const GemmParams& p_in, cudaStream_t stream, int qkv_mode, int* kernels) {
  if (kernels) *kernels = 1;
  if (p_in.M <= 0 || p_in.N <= 0 || p_in.K <= 0) return cudaSuccess;
  // Row tiles fastest (CTAs running together share W's tiles through L2), unless A is
  // both the larger operand and too large to stay in L2 between column tiles (above
  // 48 MB): then column tiles run fastest, so that A is read from memory once.  On the
  // fc2 product at 448x448 x 8 (A = 84 MB) this takes DRAM traffic from 223 to 130 MB
  // per launch at the same time (ncu); smaller A keeps the other order, which measured
  // 1-2% faster there.
  GemmParams p = p_in;
  const double a_bytes = 2.0 * p.M * p.K, w_bytes = 2.0 * p.N * p.K;
  p.n_fastest = a_bytes > w_bytes && a_bytes > 48e6 ? 1 : 0;
  // Pairs of CTAs (256-row tiles) once there are enough rows to keep them busy.
  const bool pair = p.M >= 1024;
  if (qkv_mode) {
    if (p.head_dim == 80 && p.sections[0] == 16 && p.sections[1] == 32 && p.sections[2] == 32)
      return pair ? launch_pair<240, Rope80>(p, stream) : launch_one<240, Rope80>(p, stream);
    if (p.head_dim == 32 && p.sections[0] == 8 && p.sections[1] == 12 && p.sections[2] == 12)
      return launch_one<256, Rope32>(p, stream);
    return cudaErrorNotSupported;
  }
  if (pair) {
    const int pairs = device_sm_count() / 2;
    const int mt = (p.M + 2 * kBM - 1) / (2 * kBM);
    // 256-wide tiles whose last round a split-K tail fills
    if (split_factor(p, mt * ((p.N + 255) / 256), pairs, 256) > 1) return launch_pair<256, Rope0>(p, stream, kernels);
    // otherwise 224-wide tiles when they fill the last round of CTA pairs clearly better
    // than 256-wide ones (measured on B200 for short-K, 1280-wide outputs such as the
    // attention output projection of 8 images at 448x448)
    if (p.K <= 2048) {
      auto eff = [&](int bn) {
        const int nt = (p.N + bn - 1) / bn;
        const long tiles = static_cast<long>(mt) * nt;
        const long waves = (tiles + pairs - 1) / pairs;
        return (static_cast<double>(tiles) / (waves * pairs)) * (static_cast<double>(p.N) / (nt * bn));
      };
      if (eff(224) * 0.93 > eff(256)) return launch_pair<224, Rope0>(p, stream, kernels);
    }
    return launch_pair<256, Rope0>(p, stream, kernels);
  }
  // Wide tiles when they still fill the SMs; narrower ones for small problems.
  const int sms = device_sm_count();
  const long tiles256 = static_cast<long>((p.M + kBM - 1) / kBM) * ((p.N + 255) / 256);
  if (tiles256 >= sms || p.N > 256 * 8) return launch_one<256, Rope0>(p, stream);
  return launch_one<128, Rope0>(p, stream);
}

unsigned int gemm_read_clear_error(cudaStream_t stream) {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_gemm_err, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return 0;
  cudaStreamSynchronize(stream);
  if (v) {
    cudaMemcpyToSymbolAsync(g_gemm_err, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    cudaStreamSynchronize(stream);
  }
  return v;
}

}  // namespace vt
