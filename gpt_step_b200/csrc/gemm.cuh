// tcgen05 GEMM for the dense contractions of the GPT-2 step (sm_100a).
//
//   D[M, N] = sum_k A(m, k) * B(n, k)          bf16 inputs, fp32 accumulation
//
// Operands are staged by TMA into 128-byte-swizzled shared memory and fed to
// tcgen05.mma (cta_group::1, M = 128, N = BN, K = 16 per instruction) with the
// accumulator in tensor memory. Either operand may be K-major (row-major with
// the reduction contiguous) or MN-major (the reduction is the strided index),
// which covers the three products of a linear layer without transposes:
//   forward   out  = inp . W^T    A = inp  [M, K] K-major,  B = W    [N, K] K-major
//   dgrad     din  = dout . W     A = dout [M, K] K-major,  B = W^T: W [K, N] MN-major
//   wgrad     dW  += dout^T . inp A = dout^T: dout [K, M] MN-major, B = inp [K, N] MN-major
//
// Kernel organisation (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: fills a ring of STAGES shared-memory stages
//   warp 1      allocates 2*BN tensor-memory columns; lane 0 issues the MMAs
//   warps 2..5  epilogue: tcgen05.ld the accumulator, fuse bias / residual /
//               GELU / GELU' / fp32 accumulation, store to global memory
// Two accumulator buffers in tensor memory let the epilogue of tile i overlap
// the main loop of tile i+1. No cluster multicast is used anywhere.
#pragma once
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"

namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;  // bf16 elements per 128-byte swizzle row
constexpr int UMMA_K = 16;
constexpr int kThreads = 192;

enum Epi : int {
  EPI_STORE = 0,    // out = bf16(acc [+ bias])
  EPI_RESID = 1,    // out = bf16(acc + bias + aux)            (residual add)
  EPI_GELU = 2,     // out = bf16(acc + bias); out2 = bf16(GELU(acc + bias))
  EPI_DGELU = 3,    // out = bf16(acc * GELU'(aux))
  EPI_ACC_F32 = 4,  // outf += acc (fp32; atomic when the reduction is split)
  EPI_LSE = 5,      // pair kernel only: out = bf16(acc), and per row and half tile the
                    // running (max, sum of 2^) of log2(e) * out over columns < lse_V
  EPI_LSE_ONLY = 6, // pair kernel only: the partials of EPI_LSE and the row's target logit
                    // bf16(acc)[row, lse_tgt[row]] into lse_tgt_val[row]; nothing else stored
  EPI_GELU_D = 7,   // pair kernel only: x = acc + bias; out = bf16(GELU'(x)); out2 = bf16(GELU(x))
  EPI_DMUL = 8,     // pair kernel only: out = bf16(acc * aux) (aux: the saved GELU'(x))
};
// Epilogues that store a second output (through tmO2).
constexpr bool two_outputs(int epi) { return epi == EPI_GELU || epi == EPI_GELU_D; }

struct Params {
  int M, N, K;
  int num_m, num_n, splits, kb_per_split, nkb, num_tiles;
  int raster_gm;  // row tiles per raster panel (pair kernel); num_m = plain row-major order
  float* colsum;  // pair kernel, EPI_DGELU / EPI_DMUL: column sums of the (bf16) output added here, or null
  float2* lse_part;  // pair kernel, EPI_LSE: [M][lse_slots] (max, sum) partials, slot = 2 * n_tile + half
  int lse_V, lse_slots;
  const int* sched;        // pair kernel: per-pair tile lists ([pairs + 1] offsets, then tile ids), or
                           // null for the static stride (tile t on pair t mod pairs)
  const int32_t* lse_tgt;  // EPI_LSE_ONLY: target id per row (ids outside [0, lse_V) give no value)
  float* lse_tgt_val;      // EPI_LSE_ONLY: the target's (bf16-rounded) logit per row
  bf16* out;
  bf16* out2;
  int ldo;
  const bf16* aux;
  int ld_aux;
  const float* bias;
  float* outf;
  int ldf;
  int* err;
};

template <int BN>
struct Cfg {
  static constexpr int STAGES = BN >= 256 ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_BYTES = 1024;
  // per epilogue warp: two 32x32 bf16 staging buffers for each of the (up to) two outputs
  static constexpr int EPI_BYTES = 4 * 4 * 2048;
  static constexpr int SMEM = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 2 * BN;
};

// TMA store of a 32 x 32 bf16 box (64-byte swizzle) from shared memory.
GPT2_DEV void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
GPT2_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
GPT2_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
template <int N>
GPT2_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory"); }
GPT2_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Write one thread's row of 32 bf16 (16 packed words) into a 32 x 32 staging
// buffer in the 64-byte-swizzled order the TMA store expects: 16-byte chunk j
// of row r lives at r * 64 + ((j ^ ((r >> 1) & 3)) * 16).
GPT2_DEV void stage_row(uint8_t* buf, int r, const uint32_t (&w)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int pj = j ^ ((r >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + r * 64 + pj * 16) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

GPT2_DEV void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

template <int BN, bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                   const Params p) {
  using C = Cfg<BN>;
  constexpr int S = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + S * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES + C::EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* done = bars + 2 * S + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 4 * 32);
    }
    mbar_init(smem_u32(done), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI != EPI_ACC_F32) tma_prefetch_desc(&tmO);
    if (EPI == EPI_GELU) tma_prefetch_desc(&tmO2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_begin();   // set-up above overlaps the previous kernel's drain

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        const int mb = t % p.num_m;
        const int rest = t / p.num_m;
        const int nb = rest % p.num_n;
        const int sp = rest / p.num_n;
        const int kb0 = sp * p.kb_per_split;
        const int kb1 = min(p.nkb, kb0 + p.kb_per_split);
        const int m0 = mb * BM, n0 = nb * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
          const int k0 = kb * BK;
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j) tma_load_2d(sa + j * 8192, &tmA, fb, m0 + 64 * j, k0);
          } else {
            tma_load_2d(sa, &tmA, fb, k0, m0);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 8192, &tmB, fb, n0 + 64 * j, k0);
          } else {
            tma_load_2d(sb, &tmB, fb, k0, n0);
          }
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
        const int rest = t / p.num_m;
        const int sp = rest / p.num_n;
        const int kb0 = sp * p.kb_per_split;
        const int kb1 = min(p.nkb, kb0 + p.kb_per_split);
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
            const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            tc_mma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        tc_commit(smem_u32(&tfull[acc]));
      }
      // every MMA of this CTA has completed once `done` flips
      tc_commit(smem_u32(done));
      mbar_wait(smem_u32(done), 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* wbuf = epi_smem + q * 8192;  // [out b0 | out b1 | out2 b0 | out2 b1], 2 KB each
    uint32_t nstore = 0;                  // chunks this warp has staged (selects the buffer)
    int it = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++it) {
      const int mb = t % p.num_m;
      const int rest = t / p.num_m;
      const int nb = rest % p.num_n;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.err)) break;
      tc_fence_after();
      const int row0 = mb * BM + q * 32;
      const int row = row0 + lane;
      const bool row_ok = row < p.M;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        const int n = nb * BN + c;
        float v[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c, v);
        if (n >= p.N) continue;  // uniform across the warp
        if (EPI == EPI_ACC_F32) {
          if (!row_ok) continue;
          float* dst = p.outf + (size_t)row * p.ldf + n;
          if (p.splits > 1) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) red_add_v4(dst + i, v[i], v[i + 1], v[i + 2], v[i + 3]);
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
        if (EPI == EPI_STORE || EPI == EPI_RESID || EPI == EPI_GELU) {
          if (p.bias != nullptr) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + n + i));
              v[i] += b.x; v[i + 1] += b.y; v[i + 2] += b.z; v[i + 3] += b.w;
            }
          }
        }
        if ((EPI == EPI_RESID || EPI == EPI_DGELU) && row_ok) {
          const uint4* src = reinterpret_cast<const uint4*>(p.aux + (size_t)row * p.ld_aux + n);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 u = src[j];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float2 f = unpack_bf16x2(w[h]);
              const int i = j * 8 + h * 2;
              if (EPI == EPI_RESID) {
                v[i] += f.x; v[i + 1] += f.y;
              } else {
                v[i] *= gelu_grad_f(f.x); v[i + 1] *= gelu_grad_f(f.y);
              }
            }
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
        const uint32_t b = nstore & 1;
        // the store issued from this buffer two chunks ago must have read it
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        stage_row(wbuf + b * 2048, lane, pk);
        if (EPI == EPI_GELU) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(gelu_f(v[2 * i]), gelu_f(v[2 * i + 1]));
          stage_row(wbuf + 4096 + b * 2048, lane, pk);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmO, smem_u32(wbuf + b * 2048), n, row0);
          if (EPI == EPI_GELU) tma_store_2d(&tmO2, smem_u32(wbuf + 4096 + b * 2048), n, row0);
          bulk_commit();
        }
        ++nstore;
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
    }
    if (EPI != EPI_ACC_F32 && lane == 0) bulk_wait_all<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Row-major bf16 matrix [outer][inner] with row stride `ld` elements.
static bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                     uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  return encode_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, outer, ld, box_inner, box_outer, swz);
}

static int num_sms() { return device_sm_count(); }

template <int BN, bool A_MN, bool B_MN, int EPI>
static cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
                             const CUtensorMap& to2, Params p, cudaStream_t s) {
  using C = Cfg<BN>;
  auto kern = gemm_tc_kernel<BN, A_MN, B_MN, EPI>;
  static PerDeviceOnce once;  // per template instance
  const cudaError_t e = smem_optin(once, kern, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < num_sms() ? p.num_tiles : num_sms();
  launch_pdl(kern, dim3(grid), dim3(kThreads), C::SMEM, s, ta, tb, to, to2, p);
  return cudaGetLastError();
}

// Which operand arrangement a call uses.
enum Kind { FWD = 0, DGRAD = 1, WGRAD = 2 };

// One GEMM with fused epilogue.
//   FWD:   out[M,N] = A[M,K] . B[N,K]^T   A = a (ld lda), B = b (ld ldb)
//   DGRAD: out[M,N] = A[M,K] . B[K,N]     A = a [M,K], B = b stored [K,N]
//   WGRAD: outf[M,N] += A[K,M]^T . B[K,N] A = a stored [K,M], B = b stored [K,N]
// Shapes: N % 32 == 0, K % 64 == 0, MN-major extents % 64 == 0, rows 16-byte aligned.
struct Call {
  Kind kind;
  int epi;
  int M, N, K;
  const bf16* a;
  int lda;
  const bf16* b;
  int ldb;
  bf16* out;
  bf16* out2;
  int ldo;
  const bf16* aux;
  int ld_aux;
  const float* bias;
  float* outf;
  int ldf;
  int* err;
  int force_bn;      // 0: automatic
  int force_splits;  // 0: automatic
  float* colsum;     // EPI_DGELU with >= 256 rows: add the output's column sums here (else null)
  float2* lse_part;  // EPI_LSE: [M][2 * ceil(N / 256)] row partials (see Params)
  int lse_V;         // EPI_LSE: columns >= lse_V are stored but left out of the partials
  const int32_t* lse_tgt;  // EPI_LSE_ONLY (see Params)
  float* lse_tgt_val;
};

// Tile width: whole waves of 148 SMs, with 128-wide tiles charged 1.3x because a
// single-CTA 128 x 128 x 16 MMA needs ~120 B/clk of shared-memory operand
// bandwidth (near the SM's limit) against ~90 B/clk for 128 x 256 x 16.
static int choose_bn(const Call& c) {
  if (c.force_bn) return c.force_bn;
  const long m_t = (c.M + BM - 1) / BM;
  const long sms = num_sms();
  const long t256 = m_t * ((c.N + 255) / 256), t128 = m_t * ((c.N + 127) / 128);
  const double w256 = (double)((t256 + sms - 1) / sms) * 256.0;
  const double w128 = (double)((t128 + sms - 1) / sms) * 128.0 * 1.3;
  return w256 <= w128 ? 256 : 128;
}

// Split of the reduction for weight gradients (fp32 atomic accumulation): the
// smallest split that fills the waves best, keeping >= 8 k-blocks per split.
static int choose_splits(long tiles, int nkb) {
  const long sms = num_sms();
  int best = 1;
  double best_eff = 0.0;
  for (int sp = 1; sp <= 32 && nkb >= 8 * sp; ++sp) {
    const long t = tiles * sp;
    const double eff = (double)t / (double)(sms * ((t + sms - 1) / sms));
    if (eff > best_eff + 0.03) { best_eff = eff; best = sp; }
  }
  return best;
}

static int run(const Call& c, cudaStream_t s) {
  if (c.M <= 0 || c.N <= 0 || c.K <= 0 || c.epi == EPI_LSE) return GPT2_ERR_ARG;
  if (c.N % 32 || c.K % BK) return GPT2_ERR_ARG;
  // weight gradients take full-width tiles; the split of the reduction fills the waves
  const int BN = (c.kind == WGRAD && !c.force_bn && c.N % 256 == 0) ? 256 : choose_bn(c);
  if (BN != 128 && BN != 256) return GPT2_ERR_ARG;
  Params p{};
  p.M = c.M; p.N = c.N; p.K = c.K;
  p.num_m = (c.M + BM - 1) / BM;
  p.num_n = (c.N + BN - 1) / BN;
  p.nkb = c.K / BK;
  int splits = 1;
  if (c.kind == WGRAD) {
    splits = c.force_splits ? c.force_splits : choose_splits((long)p.num_m * p.num_n, p.nkb);
  } else if (c.force_splits > 1) {
    return GPT2_ERR_ARG;
  }
  p.kb_per_split = (p.nkb + splits - 1) / splits;
  p.splits = (p.nkb + p.kb_per_split - 1) / p.kb_per_split;
  p.num_tiles = p.num_m * p.num_n * p.splits;
  p.out = c.out; p.out2 = c.out2; p.ldo = c.ldo;
  p.aux = c.aux; p.ld_aux = c.ld_aux; p.bias = c.bias;
  p.outf = c.outf; p.ldf = c.ldf; p.err = c.err;

  CUtensorMap ta, tb;
  bool ok;
  if (c.kind == WGRAD) {
    if (c.M % 64 || c.N % 64) return GPT2_ERR_ARG;
    ok = make_map(&ta, c.a, c.M, c.K, c.lda, 64, 64) && make_map(&tb, c.b, c.N, c.K, c.ldb, 64, 64);
  } else if (c.kind == DGRAD) {
    if (c.N % 64) return GPT2_ERR_ARG;
    ok = make_map(&ta, c.a, c.K, c.M, c.lda, 64, BM) && make_map(&tb, c.b, c.N, c.K, c.ldb, 64, 64);
  } else {
    ok = make_map(&ta, c.a, c.K, c.M, c.lda, 64, BM) && make_map(&tb, c.b, c.K, c.N, c.ldb, 64, BN);
  }
  if (!ok) return GPT2_ERR_ARG;
  // bf16 outputs leave through TMA stores of 32 x 32 boxes (64-byte swizzle)
  CUtensorMap to, to2;
  memset(&to, 0, sizeof(to));
  memset(&to2, 0, sizeof(to2));
  if (c.epi != EPI_ACC_F32) {
    if (!make_map(&to, c.out, c.N, c.M, c.ldo, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return GPT2_ERR_ARG;
    if (c.epi == EPI_GELU && !make_map(&to2, c.out2, c.N, c.M, c.ldo, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return GPT2_ERR_ARG;
  }

  cudaError_t e = cudaErrorInvalidValue;
#define GPT2_GEMM_CASE(BNV, AMN, BMN, EPIV) \
  e = launch_tc<BNV, AMN, BMN, EPIV>(ta, tb, to, to2, p, s)
  if (c.kind == FWD) {
    switch (c.epi) {
      case EPI_STORE: if (BN == 256) GPT2_GEMM_CASE(256, false, false, EPI_STORE); else GPT2_GEMM_CASE(128, false, false, EPI_STORE); break;
      case EPI_RESID: if (BN == 256) GPT2_GEMM_CASE(256, false, false, EPI_RESID); else GPT2_GEMM_CASE(128, false, false, EPI_RESID); break;
      case EPI_GELU:  if (BN == 256) GPT2_GEMM_CASE(256, false, false, EPI_GELU);  else GPT2_GEMM_CASE(128, false, false, EPI_GELU);  break;
      default: return GPT2_ERR_ARG;
    }
  } else if (c.kind == DGRAD) {
    switch (c.epi) {
      case EPI_STORE: if (BN == 256) GPT2_GEMM_CASE(256, false, true, EPI_STORE); else GPT2_GEMM_CASE(128, false, true, EPI_STORE); break;
      case EPI_DGELU: if (BN == 256) GPT2_GEMM_CASE(256, false, true, EPI_DGELU); else GPT2_GEMM_CASE(128, false, true, EPI_DGELU); break;
      default: return GPT2_ERR_ARG;
    }
  } else {
    if (c.epi != EPI_ACC_F32) return GPT2_ERR_ARG;
    if (BN == 256) GPT2_GEMM_CASE(256, true, true, EPI_ACC_F32); else GPT2_GEMM_CASE(128, true, true, EPI_ACC_F32);
  }
#undef GPT2_GEMM_CASE
  return e == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

}  // namespace gemm
