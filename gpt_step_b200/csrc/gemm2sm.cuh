// tcgen05 GEMM on CTA pairs (cta_group::2): 256 x BN output tiles.
//
// Same contraction and epilogues as gemm::gemm_tc_kernel, but each output tile
// of 256 rows is computed by a cluster of two CTAs on two SMs: CTA r loads its
// own 128 rows of A and its half (BN/2 rows) of B, and the even CTA issues
// tcgen05.mma.cta_group::2 (M = 256, N = BN), which reads A and B from both
// CTAs' shared memory and leaves rows 128r .. 128r+127 of the accumulator in
// CTA r's tensor memory. Per SM this moves 32 KB of operands per 4 MMAs of
// 128 x BN x 16 instead of 48 KB (B is not duplicated).
//
// Synchronisation across the pair:
//   full[s]   on the even CTA only: its producer posts the expected bytes of both
//             CTAs' loads, and both CTAs' TMA loads complete on it
//   empty[s]  on both CTAs: the MMA's commit is multicast to the pair
//   tfull[a]  on both CTAs (multicast commit); tempty[a] on the even CTA only:
//             all 256 epilogue threads of the pair arrive (the odd CTA remotely)
// No TMA multicast is used: every load reads global memory into its own CTA.
#pragma once
#include <algorithm>
#include <functional>
#include <vector>

#include "gemm.cuh"

namespace gemm2 {

using gemm::BK;
using gemm::kThreads;
using gemm::Params;
using gemm::UMMA_K;

constexpr int BM_PAIR = 256;  // rows per cluster tile (128 per CTA)

constexpr int kThreads2 = 320;  // TMA, MMA, 8 epilogue warps (two per TMEM lane quarter)

// TWO_OUT: the epilogue stores two outputs (GELU(x) and its pre-activation or
// GELU'(x)); it gets two 2 KB store buffers per output and warp, paid for with
// one operand stage.
template <int BN, bool TWO_OUT = false>
struct Cfg {
  static constexpr int STAGES = TWO_OUT ? 5 : 6;
  // epilogue staging per epilogue warp: two 2 KB store buffers per output, so
  // that a chunk is staged while the previous chunk's TMA store still reads
  static constexpr int WARP_EPI_BYTES = TWO_OUT ? 8192 : 4096;
  static constexpr int EPI_BYTES = 8 * WARP_EPI_BYTES;
  static constexpr int A_BYTES = 128 * BK * 2;          // own 128 rows
  static constexpr int B_BYTES = (BN / 2) * BK * 2;     // own half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
  static constexpr int TMEM_COLS = 2 * BN;
};

GPT2_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
GPT2_DEV uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
GPT2_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
GPT2_DEV void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
GPT2_DEV void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
GPT2_DEV void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
GPT2_DEV void tc_mma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` (same offset) in every CTA of `mask` when this thread's MMAs complete.
GPT2_DEV void tc_commit2_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// TMA load into this CTA's shared memory completing bytes on an mbarrier that may
// live in the peer CTA (shared::cluster address `bar`).
GPT2_DEV void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
GPT2_DEV void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// Tile t -> (row tile, column tile, reduction split). Output tiles run in
// panels of p.raster_gm row tiles; within a panel the row tiles vary fastest,
// then the column tiles, so the pairs working at the same time share A and B
// tiles that are still in L2 (the output stream would evict A between sweeps
// of a plain row-major order).
GPT2_DEV void tile_coords(const gemm::Params& p, int t, int& mb, int& nb, int& sp) {
  const int mn = p.num_m * p.num_n;
  sp = t / mn;
  const int r = t - sp * mn;
  const int panel_tiles = p.raster_gm * p.num_n;
  const int panel = r / panel_tiles;
  const int within = r - panel * panel_tiles;
  const int rows = min(p.raster_gm, p.num_m - panel * p.raster_gm);
  mb = panel * p.raster_gm + within % rows;
  nb = within / rows;
}

// With GROUP, a second product (a weight gradient: MN-major A and B, fp32
// accumulate; maps tmA1/tmB1, parameters p1) follows the first one's tiles in
// the same persistent tile list, so its tiles fill the first one's last wave
// and both share one pipeline fill and drain.
template <int BN, bool A_MN, bool B_MN, int EPI, bool GROUP = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                    const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ Params p1) {
  using C = Cfg<BN, gemm::two_outputs(EPI)>;
  constexpr int S = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw2[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw2) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + S * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_smem + C::EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* done = bars + 2 * S + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = (rank == 0);
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int total_tiles = p.num_tiles + (GROUP ? p1.num_tiles : 0);
  // this pair's tiles: a host-built list, or every ncl-th tile from cid
  const int* sch = p.sched;
  const int k_beg = sch ? sch[cid] : cid, k_end = sch ? sch[cid + 1] : total_tiles, k_step = sch ? 1 : ncl;
  const int* sch_tiles = sch ? sch + ncl + 1 : nullptr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 2 * 8);   // one arrival per epilogue warp of the pair
    }
    mbar_init(smem_u32(done), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (GROUP) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
    if (EPI != gemm::EPI_ACC_F32 && EPI != gemm::EPI_LSE_ONLY) tma_prefetch_desc(&tmO);
    if (EPI == gemm::EPI_GELU || EPI == gemm::EPI_GELU_D) tma_prefetch_desc(&tmO2);
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up above overlaps the previous kernel's drain; operands and outputs only after it
  pdl_begin();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int k = k_beg; k < k_end && ok; k += k_step) {
        const int t = sch ? sch_tiles[k] : k;
        const bool second = GROUP && t >= p.num_tiles;
        const Params& q = second ? p1 : p;
        int mb, nb, sp;
        tile_coords(q, second ? t - p.num_tiles : t, mb, nb, sp);
        const int kb0 = sp * q.kb_per_split;
        const int kb1 = min(q.nkb, kb0 + q.kb_per_split);
        const int m0 = mb * BM_PAIR + 128 * rank;
        const int n0 = nb * BN + (BN / 2) * rank;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * C::STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
          const int k0 = kb * BK;
          if (second) {
#pragma unroll
            for (int j = 0; j < 2; ++j) tma_load_2d_pair(sa + j * 8192, &tmA1, fb, m0 + 64 * j, k0);
#pragma unroll
            for (int j = 0; j < BN / 128; ++j) tma_load_2d_pair(sb + j * 8192, &tmB1, fb, n0 + 64 * j, k0);
          } else {
            if (A_MN) {
#pragma unroll
              for (int j = 0; j < 2; ++j) tma_load_2d_pair(sa + j * 8192, &tmA, fb, m0 + 64 * j, k0);
            } else {
              tma_load_2d_pair(sa, &tmA, fb, k0, m0);
            }
            if (B_MN) {
#pragma unroll
              for (int j = 0; j < BN / 128; ++j) tma_load_2d_pair(sb + j * 8192, &tmB, fb, n0 + 64 * j, k0);
            } else {
              tma_load_2d_pair(sb, &tmB, fb, k0, n0);
            }
          }
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc0 = idesc_bf16_f32(BM_PAIR, BN, A_MN, B_MN);
      constexpr uint32_t idesc1 = idesc_bf16_f32(BM_PAIR, BN, true, true);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int k = k_beg; k < k_end && ok; k += k_step, ++it) {
        const int t = sch ? sch_tiles[k] : k;
        const bool second = GROUP && t >= p.num_tiles;
        const Params& q = second ? p1 : p;
        const int tt = second ? t - p.num_tiles : t;
        // tile bookkeeping stays off the MMA issue path: no division without a split
        const int sp = q.splits == 1 ? 0 : tt / (q.num_m * q.num_n);
        const int kb0 = sp * q.kb_per_split;
        const int kb1 = min(q.nkb, kb0 + q.kb_per_split);
        const bool a_mn = second || A_MN, b_mn = second || B_MN;
        const uint32_t idesc = second ? idesc1 : idesc0;
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint64_t ad = a_mn ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = b_mn ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            tc_mma2_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          tc_commit2_mc(smem_u32(&empty[stage]), 0x3);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        tc_commit2_mc(smem_u32(&tfull[acc]), 0x3);
      }
      tc_commit2_mc(smem_u32(done), 0x1);
      mbar_wait(smem_u32(done), 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;              // TMEM lane quarter
    const int hv = (warp - 2) >> 2;      // column half of the tile this warp drains
    uint8_t* wbuf = epi_smem + (warp - 2) * C::WARP_EPI_BYTES;
    uint32_t nstore = 0;
    int it = 0;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    // The residual / GELU' operand of a tile (this lane's row, this warp's half
    // of the columns) is prefetched into L2 one tile ahead, while the tensor
    // cores still work on the tile before it: the epilogue's operand loads then
    // wait on L2, not DRAM (with a DRAM wait per 32-column chunk the epilogue
    // outlasted the main loop of the 768 x 768 projection).
    constexpr bool kAuxPf = EPI == gemm::EPI_RESID || EPI == gemm::EPI_DGELU || EPI == gemm::EPI_DMUL;
    auto prefetch_aux = [&](int kk) {
      if (kk >= k_end) return;
      const int tn = sch ? sch_tiles[kk] : kk;
      if (GROUP && tn >= p.num_tiles) return;   // weight-gradient tiles read no operand here
      int mb, nb, sp;
      tile_coords(p, tn, mb, nb, sp);
      (void)sp;
      const int row = mb * BM_PAIR + 128 * rank + q * 32 + lane;
      const int n0 = nb * BN + hv * (BN / 2);
      if (row >= p.M || n0 >= p.N) return;
      const bf16* a = p.aux + (size_t)row * p.ld_aux + n0;
      const int ncols = min(BN / 2, p.N - n0);
      for (int c = 0; c < ncols; c += 64) prefetch_l2(a + c);    // 128-byte lines
      prefetch_l2(a + ncols - 1);
    };
    if (kAuxPf && p.aux != nullptr) prefetch_aux(k_beg);
    for (int k = k_beg; k < k_end; k += k_step, ++it) {
      const int t = sch ? sch_tiles[k] : k;
      const bool second = GROUP && t >= p.num_tiles;
      int mb, nb, sp;
      tile_coords(second ? p1 : p, second ? t - p.num_tiles : t, mb, nb, sp);
      (void)sp;
      if (kAuxPf && p.aux != nullptr) prefetch_aux(k + k_step);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.err)) break;
      tc_fence_after();
      const int row0 = mb * BM_PAIR + 128 * rank + q * 32;
      const int row = row0 + lane;
      const bool row_ok = row < (second ? p1.M : p.M);
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      if (second) {
        // weight-gradient tile: fp32 accumulate (vector atomics when K is split)
#pragma unroll 1
        for (int c = hv * (BN / 2); c < (hv + 1) * (BN / 2); c += 32) {
          float v[32];
          tmem_ld32(t_row + c, v);
          const int n = nb * BN + c;
          if (n >= p1.N || !row_ok) continue;
          float* dst = p1.outf + (size_t)row * p1.ldf + n;
          if (p1.splits > 1) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) gemm::red_add_v4(dst + i, v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 o = *reinterpret_cast<float4*>(dst + i);
              o.x += v[i]; o.y += v[i + 1]; o.z += v[i + 2]; o.w += v[i + 3];
              *reinterpret_cast<float4*>(dst + i) = o;
            }
          }
        }
      } else {
        // Chunk c + 32 is read from tensor memory, and its bias / aux operands
        // from global memory, while chunk c is processed: the epilogue of a tile
        // then runs at about the pace of the next tile's main loop.
        constexpr bool kBias = EPI == gemm::EPI_STORE || EPI == gemm::EPI_RESID || EPI == gemm::EPI_GELU ||
                               EPI == gemm::EPI_LSE || EPI == gemm::EPI_GELU_D;
        constexpr bool kTwoOut = EPI == gemm::EPI_GELU || EPI == gemm::EPI_GELU_D;
        constexpr bool kLse = EPI == gemm::EPI_LSE || EPI == gemm::EPI_LSE_ONLY;
        constexpr bool kStore = EPI != gemm::EPI_LSE_ONLY;
        // EPI_LSE_ONLY: the row's target id, if it falls in this half tile (else -1)
        int tgt_col = -1;
        if (EPI == gemm::EPI_LSE_ONLY && row_ok) {
          const int tg = __ldg(p.lse_tgt + row) - (nb * BN + hv * (BN / 2));
          if (tg >= 0 && tg < BN / 2 && nb * BN + hv * (BN / 2) + tg < p.lse_V) tgt_col = tg;
        }
        // EPI_LSE: this row's running max (log2 units) and sum of 2^(y - max) over the half tile
        float lse_m = -INFINITY, lse_s = 0.f;
        constexpr bool kAux = EPI == gemm::EPI_RESID || EPI == gemm::EPI_DGELU || EPI == gemm::EPI_DMUL;
        const bool has_bias = kBias && p.bias != nullptr;
        const int c_beg = hv * (BN / 2), c_end = (hv + 1) * (BN / 2);
        uint32_t vr[32];
        float4 bn4[8];
        uint4 an4[4];
        auto fetch = [&](int c) {
          tmem_ld32_async(t_row + c, vr);
          const int n = nb * BN + c;
          if (n < p.N) {
            if (has_bias) {
#pragma unroll
              for (int i = 0; i < 8; ++i) bn4[i] = __ldg(reinterpret_cast<const float4*>(p.bias + n) + i);
            }
            if (kAux) {
              // coalesced: lane l loads 16-byte chunk l & 3 of the warp's rows
              // (l >> 2) + 8 i, eight 64-byte row segments per instruction; the
              // staging box turns them into one row per lane when consumed
              const int j = lane & 3;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int rr = row0 + (lane >> 2) + 8 * i;
                an4[i] = rr < p.M ? __ldcs(reinterpret_cast<const uint4*>(p.aux + (size_t)rr * p.ld_aux + n + 8 * j))
                                  : make_uint4(0u, 0u, 0u, 0u);
              }
            }
          }
        };
        fetch(c_beg);
#pragma unroll 1
        for (int c = c_beg; c < c_end; c += 32) {
          const int n = nb * BN + c;
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(vr[i]);
          // consume this chunk's bias / aux registers, then start the next chunk's loads
          // (paired fp32 operations: two columns per instruction)
          if (n < p.N && has_bias) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 lo = f2_add(make_float2(v[4 * i], v[4 * i + 1]), make_float2(bn4[i].x, bn4[i].y));
              const float2 hi = f2_add(make_float2(v[4 * i + 2], v[4 * i + 3]), make_float2(bn4[i].z, bn4[i].w));
              v[4 * i] = lo.x; v[4 * i + 1] = lo.y; v[4 * i + 2] = hi.x; v[4 * i + 3] = hi.y;
            }
          }
          if (kAux && n < p.N) {
            // through this chunk's staging box (once the TMA store from it two
            // chunks ago has read it): written as loaded, read back one row per lane
            uint8_t* box = wbuf + (nstore & 1) * 2048;
            if (lane == 0) gemm::bulk_wait_read<1>();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = (lane >> 2) + 8 * i, j = lane & 3;
              *reinterpret_cast<uint4*>(box + r * 64 + ((j ^ ((r >> 1) & 3)) << 4)) = an4[i];
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              an4[j] = *reinterpret_cast<const uint4*>(box + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4));
            __syncwarp();
          }
          if (kAux && n < p.N && row_ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t w[4] = {an4[j].x, an4[j].y, an4[j].z, an4[j].w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const float2 f = unpack_bf16x2(w[h]);
                const int i = j * 8 + h * 2;
                float2 r = make_float2(v[i], v[i + 1]);
                if (EPI == gemm::EPI_RESID) {
                  r = f2_add(r, f);
                } else if (EPI == gemm::EPI_DMUL) {
                  r = f2_mul(r, f);
                } else {
                  r = f2_mul(r, make_float2(gelu_grad_f(f.x), gelu_grad_f(f.y)));
                }
                v[i] = r.x; v[i + 1] = r.y;
              }
            }
          }
          if (c + 32 < c_end) fetch(c + 32);
          if (n >= p.N) continue;
          if (EPI == gemm::EPI_ACC_F32) {
            if (!row_ok) continue;
            float* dst = p.outf + (size_t)row * p.ldf + n;
            if (p.splits > 1) {
#pragma unroll
              for (int i = 0; i < 32; i += 4) gemm::red_add_v4(dst + i, v[i], v[i + 1], v[i + 2], v[i + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                float4 o = *reinterpret_cast<float4*>(dst + i);
                o.x += v[i]; o.y += v[i + 1]; o.z += v[i + 2]; o.w += v[i + 3];
                *reinterpret_cast<float4*>(dst + i) = o;
              }
            }
            continue;
          }
          uint32_t pk[16];
          if (EPI == gemm::EPI_GELU_D) {
            // first output GELU'(x) (what the backward multiplies by), then GELU(x) into v
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float2 g, d;
              gelu_and_grad_f2(make_float2(v[2 * i], v[2 * i + 1]), g, d);
              pk[i] = pack_bf16x2(d.x, d.y);
              v[2 * i] = g.x;
              v[2 * i + 1] = g.y;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          }
          if (kLse) {
            // over the stored bf16 values f: chunk max by a bf16x2 tree (exact, and
            // max(f) * log2(e) rounds to the max of the scaled values), then the sum
            // of 2^(f log2(e) - max) in four independent accumulators
            const float kL2e = 1.4426950408889634f;
            float cm;
            float f[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 u = unpack_bf16x2(pk[i]);
              f[2 * i] = u.x;
              f[2 * i + 1] = u.y;
            }
            if (n + 32 <= p.lse_V) {
              __nv_bfloat162 h[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) h[i] = *reinterpret_cast<const __nv_bfloat162*>(&pk[i]);
#pragma unroll
              for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) h[i] = __hmax2(h[i], h[i + w]);
              const float2 hm = __bfloat1622float2(h[0]);
              cm = fmaxf(hm.x, hm.y) * kL2e;
            } else {
              cm = -INFINITY;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                if (n + i >= p.lse_V) f[i] = -INFINITY;   // padded ids: 2^-inf = 0
                cm = fmaxf(cm, f[i]);
              }
              cm *= kL2e;
            }
            if (cm > lse_m) {
              lse_s *= ex2_approx(lse_m - cm);
              lse_m = cm;
            }
            if (cm != -INFINITY) {
              // two columns per paired fp32 instruction, four independent sums
              const float2 l2e2 = make_float2(kL2e, kL2e), nm2 = make_float2(-lse_m, -lse_m);
              float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 y = f2_fma(make_float2(f[2 * i], f[2 * i + 1]), l2e2, nm2);
                const float2 e = make_float2(ex2_approx(y.x), ex2_approx(y.y));
                if (i & 1) a1 = f2_add(a1, e);
                else a0 = f2_add(a0, e);
              }
              lse_s += (a0.x + a0.y) + (a1.x + a1.y);
            }
            if (EPI == gemm::EPI_LSE_ONLY) {
              const int k = tgt_col - (c - c_beg);
              if (k >= 0 && k < 32) {
                float tv = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) tv = (i == k) ? f[i] : tv;
                p.lse_tgt_val[row] = tv;
              }
            }
          }
          if (!kStore) continue;
          // alternate two buffers per output: the stores of the chunk before the
          // previous one (one commit group per chunk) must have read theirs
          const uint32_t b = nstore & 1;
          if (lane == 0) gemm::bulk_wait_read<1>();
          __syncwarp();
          if (!row_ok) {   // rows past M: the store leaves them out; the column sums must see 0
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
          gemm::stage_row(wbuf + b * 2048, lane, pk);
          if ((EPI == gemm::EPI_DGELU || EPI == gemm::EPI_DMUL) && p.colsum != nullptr) {
            // column sums of the stored (bf16) values over this warp's 32 rows, read
            // back from the staged box (rows of 64 bytes, 16-byte chunks swizzled by
            // (row >> 1) & 3; rows past M staged as zeros): lane l adds column pair
            // l & 15 over rows 16 (l >> 4) .. +15, then the two row halves combine
            __syncwarp();
            const uint8_t* box = wbuf + b * 2048;
            const int cp = lane & 15, r0h = (lane >> 4) * 16;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
              const int r = r0h + rr;
              const uint32_t w = *reinterpret_cast<const uint32_t*>(
                  box + r * 64 + (((cp >> 2) ^ ((r >> 1) & 3)) << 4) + (cp & 3) * 4);
              const float2 f = unpack_bf16x2(w);
              s0 += f.x;
              s1 += f.y;
            }
            s0 += __shfl_xor_sync(0xffffffffu, s0, 16);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 16);
            if (lane < 16) {
              atomicAdd(p.colsum + n + 2 * cp, s0);
              atomicAdd(p.colsum + n + 2 * cp + 1, s1);
            }
          }
          if (kTwoOut) {
            if (EPI == gemm::EPI_GELU_D) {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);   // GELU(x), formed above
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(gelu_f(v[2 * i]), gelu_f(v[2 * i + 1]));
            }
            gemm::stage_row(wbuf + 4096 + b * 2048, lane, pk);
          }
          gemm::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            gemm::tma_store_2d(&tmO, smem_u32(wbuf + b * 2048), n, row0);
            if (kTwoOut) gemm::tma_store_2d(&tmO2, smem_u32(wbuf + 4096 + b * 2048), n, row0);
            gemm::bulk_commit();
          }
          ++nstore;
        }
        if (kLse && row_ok) p.lse_part[(size_t)row * p.lse_slots + 2 * nb + hv] = make_float2(lse_m, lse_s);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc ? tempty_leader1 : tempty_leader0);
    }
    if (EPI != gemm::EPI_ACC_F32 && EPI != gemm::EPI_LSE_ONLY && lane == 0) gemm::bulk_wait_all<0>();
  }

  tc_fence_before();
  cluster_sync();  // no CTA leaves while its pair may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, C::TMEM_COLS);
  }
}

template <int BN, bool A_MN, bool B_MN, int EPI, bool GROUP = false>
static cudaError_t launch_tc2(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
                              const CUtensorMap& to2, const Params& p, cudaStream_t s,
                              const CUtensorMap* ta1 = nullptr, const CUtensorMap* tb1 = nullptr,
                              const Params* p1 = nullptr) {
  using C = Cfg<BN, gemm::two_outputs(EPI)>;
  auto kern = gemm_tc2_kernel<BN, A_MN, B_MN, EPI, GROUP>;
  static PerDeviceOnce once;  // per template instance
  const cudaError_t e = smem_optin(once, kern, C::SMEM);
  if (e != cudaSuccess) return e;
  Params q1{};
  if (GROUP) q1 = *p1;
  const int total = p.num_tiles + q1.num_tiles;
  const int pairs = gemm::num_sms() / 2;
  // a planned schedule has one tile list per pair, some possibly empty
  const int grid = 2 * ((p.sched != nullptr || total >= pairs) ? pairs : total);
  return launch_pdl(kern, dim3(grid), dim3(kThreads2), C::SMEM, s, ta, tb, to, to2, p, GROUP ? *ta1 : ta,
                    GROUP ? *tb1 : tb, q1);
}

}  // namespace gemm2

namespace gemm2 {

// Entry point for every GEMM of the step: CTA pairs for tiles of 256 x 256 when
// the output has at least 256 rows and 256-wide tiles are chosen, otherwise the
// single-CTA kernel (gemm::run).
// Row tiles per raster panel (measured on the step's shapes: 16 for forward and
// dgrad GEMMs, 8 for weight gradients; plain row-major order was 9-18% slower
// on outputs 768 wide).
constexpr int kRasterRows = 16, kRasterRowsWgrad = 8;

// Whether run() takes the pair kernel for this call (the only one with fused
// column sums).
static bool uses_pair(const gemm::Call& c) {
  using namespace gemm;
  const int BN = (c.kind == WGRAD && !c.force_bn && c.N % 256 == 0) ? 256 : choose_bn(c);
  return BN == 256 && c.M >= BM_PAIR && c.force_bn != 128;
}

// Tile parameters and tensor maps of one pair-kernel product. splits > 0 forces
// the reduction split of a weight gradient.
static int prepare(const gemm::Call& c, int splits_forced, Params& p, CUtensorMap& ta, CUtensorMap& tb,
                   CUtensorMap& to, CUtensorMap& to2) {
  using namespace gemm;
  const int BN = 256;
  p = Params{};
  p.M = c.M; p.N = c.N; p.K = c.K;
  p.num_m = (c.M + BM_PAIR - 1) / BM_PAIR;
  p.num_n = (c.N + BN - 1) / BN;
  p.nkb = c.K / BK;
  int splits = 1;
  if (c.kind == WGRAD) {
    // waves of SM pairs: the split search sees pair tiles against 74 pairs
    if (splits_forced > 0) {
      splits = splits_forced;
    } else if (c.force_splits) {
      splits = c.force_splits;
    } else {
      const long pairs = num_sms() / 2;
      double best_eff = 0.0;
      for (int sp = 1; sp <= 32 && p.nkb >= 8 * sp; ++sp) {
        const long t = (long)p.num_m * p.num_n * sp;
        const double eff = (double)t / (double)(pairs * ((t + pairs - 1) / pairs));
        if (eff > best_eff + 0.03) { best_eff = eff; splits = sp; }
      }
    }
  } else if (c.force_splits > 1) {
    return GPT2_ERR_ARG;
  }
  p.kb_per_split = (p.nkb + splits - 1) / splits;
  p.splits = (p.nkb + p.kb_per_split - 1) / p.kb_per_split;
  p.num_tiles = p.num_m * p.num_n * p.splits;
  p.raster_gm = std::min(p.num_m, c.kind == WGRAD ? kRasterRowsWgrad : kRasterRows);
  p.colsum = (c.epi == EPI_DGELU || c.epi == EPI_DMUL) ? c.colsum : nullptr;
  if (c.epi == EPI_LSE || c.epi == EPI_LSE_ONLY) {
    if (c.kind != FWD || !c.lse_part || c.lse_V <= 0 || c.lse_V > c.N) return GPT2_ERR_ARG;
    p.lse_part = c.lse_part;
    p.lse_V = c.lse_V;
    p.lse_slots = 2 * p.num_n;
    if (c.epi == EPI_LSE_ONLY) {
      if (!c.lse_tgt || !c.lse_tgt_val) return GPT2_ERR_ARG;
      p.lse_tgt = c.lse_tgt;
      p.lse_tgt_val = c.lse_tgt_val;
    }
  }
  p.out = c.out; p.out2 = c.out2; p.ldo = c.ldo;
  p.aux = c.aux; p.ld_aux = c.ld_aux; p.bias = c.bias;
  p.outf = c.outf; p.ldf = c.ldf; p.err = c.err;

  memset(&to, 0, sizeof(to));
  memset(&to2, 0, sizeof(to2));
  bool ok;
  if (c.kind == WGRAD) {
    if (c.M % 64 || c.N % 64) return GPT2_ERR_ARG;
    ok = make_map(&ta, c.a, c.M, c.K, c.lda, 64, 64) && make_map(&tb, c.b, c.N, c.K, c.ldb, 64, 64);
  } else if (c.kind == DGRAD) {
    if (c.N % 64) return GPT2_ERR_ARG;
    ok = make_map(&ta, c.a, c.K, c.M, c.lda, 64, 128) && make_map(&tb, c.b, c.N, c.K, c.ldb, 64, 64);
  } else {
    ok = make_map(&ta, c.a, c.K, c.M, c.lda, 64, 128) && make_map(&tb, c.b, c.K, c.N, c.ldb, 64, BN / 2);
  }
  if (!ok) return GPT2_ERR_ARG;
  if (c.epi != EPI_ACC_F32 && c.epi != EPI_LSE_ONLY) {
    if (!make_map(&to, c.out, c.N, c.M, c.ldo, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return GPT2_ERR_ARG;
    if ((c.epi == EPI_GELU || c.epi == EPI_GELU_D) &&
        !make_map(&to2, c.out2, c.N, c.M, c.ldo, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return GPT2_ERR_ARG;
  }
  return GPT2_OK;
}

static int run(const gemm::Call& c, cudaStream_t s) {
  using namespace gemm;
  if (c.M <= 0 || c.N <= 0 || c.K <= 0) return GPT2_ERR_ARG;
  if (c.N % 32 || c.K % BK) return GPT2_ERR_ARG;
  const bool pair = uses_pair(c);
  if (!pair && c.colsum) return GPT2_ERR_ARG;   // fused column sums need the pair kernel
  if (!pair && (c.epi == EPI_GELU_D || c.epi == EPI_DMUL)) return GPT2_ERR_ARG;
  if (!pair) return gemm::run(c, s);   // refuses EPI_LSE
  Params p;
  CUtensorMap ta, tb, to, to2;
  const int st = prepare(c, 0, p, ta, tb, to, to2);
  if (st != GPT2_OK) return st;
  cudaError_t e = cudaErrorInvalidValue;
  if (c.kind == FWD) {
    switch (c.epi) {
      case EPI_STORE: e = launch_tc2<256, false, false, EPI_STORE>(ta, tb, to, to2, p, s); break;
      case EPI_RESID: e = launch_tc2<256, false, false, EPI_RESID>(ta, tb, to, to2, p, s); break;
      case EPI_GELU: e = launch_tc2<256, false, false, EPI_GELU>(ta, tb, to, to2, p, s); break;
      case EPI_GELU_D: e = launch_tc2<256, false, false, EPI_GELU_D>(ta, tb, to, to2, p, s); break;
      case EPI_LSE: e = launch_tc2<256, false, false, EPI_LSE>(ta, tb, to, to2, p, s); break;
      case EPI_LSE_ONLY: e = launch_tc2<256, false, false, EPI_LSE_ONLY>(ta, tb, to, to2, p, s); break;
      default: return GPT2_ERR_ARG;
    }
  } else if (c.kind == DGRAD) {
    switch (c.epi) {
      case EPI_STORE: e = launch_tc2<256, false, true, EPI_STORE>(ta, tb, to, to2, p, s); break;
      case EPI_DGELU: e = launch_tc2<256, false, true, EPI_DGELU>(ta, tb, to, to2, p, s); break;
      case EPI_DMUL: e = launch_tc2<256, false, true, EPI_DMUL>(ta, tb, to, to2, p, s); break;
      default: return GPT2_ERR_ARG;
    }
  } else {
    if (c.epi != EPI_ACC_F32) return GPT2_ERR_ARG;
    e = launch_tc2<256, true, true, EPI_ACC_F32>(ta, tb, to, to2, p, s);
  }
  return e == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

// Tile plan of a grouped launch whose schedule is built once on the host and
// kept in device memory by the caller: the weight gradient's reduction split
// and, per SM pair, the list of tiles it runs.
struct GroupPlan {
  int splits1 = 0;              // 0: no plan (static stride, split chosen per call)
  std::vector<int> table;       // [pairs + 1] offsets, then tile ids
  long makespan = 0;            // estimated k-block units of the busiest pair
};

// Longest-processing-time-first assignment: tiles in order of decreasing cost
// (k-blocks plus an epilogue allowance, plus an atomic-pass allowance for split
// weight-gradient tiles), each to the least loaded pair; each pair then runs its
// tiles in increasing tile order, so pairs working at the same time stay on
// nearby raster panels. The split of the weight gradient is the one with the
// smallest estimated makespan.
static GroupPlan plan_group(const gemm::Call& c0, const gemm::Call& c1, int pairs) {
  using namespace gemm;
  constexpr int kEpi = 2, kAtomic = 8;
  GroupPlan best;
  const long tiles0 = (long)((c0.M + BM_PAIR - 1) / BM_PAIR) * ((c0.N + 255) / 256);
  const int cost0 = c0.K / BK + kEpi;
  const int nkb1 = c1.K / BK;
  const long tiles1 = (long)((c1.M + BM_PAIR - 1) / BM_PAIR) * (c1.N / 256);
  for (int sp = 1; sp <= 32 && nkb1 >= 8 * sp; ++sp) {
    const int kbps = (nkb1 + sp - 1) / sp;
    const int nsp = (nkb1 + kbps - 1) / kbps;
    if (nsp != sp) continue;
    const int cost1 = kbps + kEpi + (nsp > 1 ? kAtomic : 0);
    const long n = tiles0 + tiles1 * nsp;
    // tiles of the costlier product first; within a product in tile order
    std::vector<std::pair<long, int>> heap;   // (load, pair) min-heap
    for (int i = 0; i < pairs; ++i) heap.push_back({0L, i});
    std::vector<std::vector<int>> lists(pairs);
    auto assign = [&](long first, long count, int cost) {
      for (long t = first; t < first + count; ++t) {
        std::pop_heap(heap.begin(), heap.end(), std::greater<>());
        heap.back().first += cost;
        lists[heap.back().second].push_back((int)t);
        std::push_heap(heap.begin(), heap.end(), std::greater<>());
      }
    };
    if (cost0 >= cost1) { assign(0, tiles0, cost0); assign(tiles0, tiles1 * nsp, cost1); }
    else { assign(tiles0, tiles1 * nsp, cost1); assign(0, tiles0, cost0); }
    long mk = 0;
    for (auto& h : heap) mk = std::max(mk, h.first);
    if (best.splits1 == 0 || mk < best.makespan) {
      best.splits1 = nsp;
      best.makespan = mk;
      best.table.assign(pairs + 1 + n, 0);
      int o = 0;
      for (int i = 0; i < pairs; ++i) {
        std::sort(lists[i].begin(), lists[i].end());
        best.table[i] = o;
        for (int t : lists[i]) best.table[pairs + 1 + o++] = t;
      }
      best.table[pairs] = o;
    }
  }
  return best;
}

// A layer's input gradient (dgrad, c0) and weight gradient (wgrad, c1) in one
// launch: c1's tiles follow c0's in the persistent tile list, its reduction
// split chosen so that its tiles carry about as many k-blocks as c0's. Falls
// back to two launches when either product does not take the pair kernel.
// With a plan (its split and its per-pair tile lists already in device memory
// at dev_sched), the pairs run the planned lists.
// Whether a dgrad (c0) and a wgrad (c1) can share one launch of the pair kernel.
static bool groupable(const gemm::Call& c0, const gemm::Call& c1) {
  using namespace gemm;
  return c0.kind == DGRAD && c1.kind == WGRAD && c1.epi == EPI_ACC_F32 && c0.M > 0 && c0.N % 32 == 0 &&
         c0.K % BK == 0 && c1.K % BK == 0 && c1.K > 0 && uses_pair(c0) && uses_pair(c1) && c1.N % 256 == 0;
}

static int run_group(const gemm::Call& c0, const gemm::Call& c1, cudaStream_t s, int* launches,
                     int* splits_out = nullptr, int plan_splits = 0, const int* dev_sched = nullptr) {
  using namespace gemm;
  const bool ok_shapes = groupable(c0, c1);
  *launches = ok_shapes ? 1 : 2;
  if (splits_out) *splits_out = 0;
  if (!ok_shapes) {
    const int st = gemm2::run(c0, s);
    return st != GPT2_OK ? st : gemm2::run(c1, s);
  }
  Params p0, p1;
  CUtensorMap ta0, tb0, to0, to20, ta1, tb1, to1, to21;
  int st = prepare(c0, 0, p0, ta0, tb0, to0, to20);
  if (st != GPT2_OK) return st;
  // The wgrad split that minimises the estimated finish time of the busiest SM
  // pair under the round-robin tile order: a tile costs its k-blocks plus an
  // epilogue allowance, a split tile a further allowance for its fp32 atomic pass.
  const int nkb1 = c1.K / BK;
  const long tiles1 = (long)((c1.M + BM_PAIR - 1) / BM_PAIR) * (c1.N / 256);
  const int pairs = num_sms() / 2;
  constexpr int kEpi = 2, kAtomic = 8;
  int splits1 = 1;
  long best = -1;
  std::vector<long> load(pairs);
  for (int sp = 1; sp <= 32 && nkb1 >= 8 * sp; ++sp) {
    const int kbps = (nkb1 + sp - 1) / sp;
    const int nsp = (nkb1 + kbps - 1) / kbps;
    std::fill(load.begin(), load.end(), 0L);
    long t = 0;
    for (long i = 0; i < p0.num_tiles; ++i, ++t) load[t % pairs] += p0.nkb + kEpi;
    for (long i = 0; i < tiles1 * nsp; ++i, ++t) load[t % pairs] += kbps + kEpi + (nsp > 1 ? kAtomic : 0);
    const long mk = *std::max_element(load.begin(), load.end());
    if (best < 0 || mk < best) { best = mk; splits1 = nsp; }
  }
  if (dev_sched != nullptr) {
    if (plan_splits <= 0) return GPT2_ERR_ARG;
    splits1 = plan_splits;
  }
  st = prepare(c1, splits1, p1, ta1, tb1, to1, to21);
  if (st != GPT2_OK) return st;
  if (dev_sched != nullptr && p1.splits != plan_splits) return GPT2_ERR_ARG;
  p0.sched = dev_sched;
  if (splits_out) *splits_out = p1.splits;
  cudaError_t e = cudaErrorInvalidValue;
  switch (c0.epi) {
    case EPI_STORE: e = launch_tc2<256, false, true, EPI_STORE, true>(ta0, tb0, to0, to20, p0, s, &ta1, &tb1, &p1); break;
    case EPI_DGELU: e = launch_tc2<256, false, true, EPI_DGELU, true>(ta0, tb0, to0, to20, p0, s, &ta1, &tb1, &p1); break;
    case EPI_DMUL: e = launch_tc2<256, false, true, EPI_DMUL, true>(ta0, tb0, to0, to20, p0, s, &ta1, &tb1, &p1); break;
    default: return GPT2_ERR_ARG;
  }
  return e == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

}  // namespace gemm2
