// Causal flash attention, forward and backward, for head sizes 32 and 64.
//
// Scaled dot-product attention with a causal mask (grow_a_language_model_intro,
// activities 5-6: Q.K^T/sqrt(d), causal mask, softmax; heads split), computed
// without materialising the T x T scores: the forward keeps a running row
// maximum and sum (online softmax) over 64-key blocks and saves the per-row
// log-sum-exp; the backward recomputes the probabilities from it.
//
// Layout: qkv is bf16 [B, T, 3C] with q | k | v and heads contiguous inside each
// (head h occupies columns h*hd .. h*hd+hd-1 of its third); the output is bf16
// [B, T, C]; lse is fp32 [B, H, T] (natural log of the scaled scores).
//
// The products run on the bf16 tensor cores through mma.sync m16n8k16 with
// fp32 accumulation; fragments move between shared memory and registers with
// ldmatrix. Each CTA has 4 warps; a warp owns 16 rows of a 64-row block.
#pragma once
#include "common.cuh"

namespace attn {

constexpr int BLK = 64;

GPT2_DEV void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

GPT2_DEV void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
GPT2_DEV void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

GPT2_DEV void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
GPT2_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
GPT2_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared tile of 64 rows x HD bf16, rows padded by 8 elements (16 bytes) so that
// ldmatrix row addresses fall in distinct banks.
template <int HD>
struct Tile {
  static constexpr int LD = HD + 8;
  static constexpr int BYTES = BLK * LD * 2;
};

// Copy 64 rows of HD elements (row stride ld elements) from global to a padded tile.
template <int HD>
GPT2_DEV void load_tile(bf16* s, const bf16* g, int ld) {
  constexpr int VPR = HD / 8;  // 16-byte vectors per row
  for (int i = threadIdx.x; i < BLK * VPR; i += 128) {
    const int r = i / VPR, c = (i % VPR) * 8;
    cp_async16(smem_u32(s + r * Tile<HD>::LD + c), g + (size_t)r * ld + c);
  }
}

// A fragment (16 x 16) at rows r0.., cols c0.. of a row-major padded tile.
template <int LD>
GPT2_DEV void frag_a(const bf16* s, int r0, int c0, uint32_t (&a)[4]) {
  const int l = lane_id();
  const int r = r0 + (l & 7) + 8 * ((l >> 3) & 1);
  const int c = c0 + 8 * (l >> 4);
  ldsm_x4(smem_u32(s + r * LD + c), a[0], a[1], a[2], a[3]);
}
// A fragment (16 x 16) of the TRANSPOSE of a row-major tile: A[m][k] = s[k0+k][m0+m].
template <int LD>
GPT2_DEV void frag_a_t(const bf16* s, int m0, int k0, uint32_t (&a)[4]) {
  const int l = lane_id();
  const int r = k0 + (l & 7) + 8 * (l >> 4);
  const int c = m0 + 8 * ((l >> 3) & 1);
  ldsm_x4_t(smem_u32(s + r * LD + c), a[0], a[1], a[2], a[3]);
}
// B fragments for two n8 tiles (n0..n0+15) and k16 (k0..): B[k][n] = s[n][k]
// (tile stored with n as the row). b[0],b[1] -> tile n0; b[2],b[3] -> tile n0+8.
template <int LD>
GPT2_DEV void frag_b_nk(const bf16* s, int n0, int k0, uint32_t (&b)[4]) {
  const int l = lane_id();
  const int r = n0 + (l & 7) + 8 * (l >> 4);
  const int c = k0 + 8 * ((l >> 3) & 1);
  ldsm_x4(smem_u32(s + r * LD + c), b[0], b[1], b[2], b[3]);
}
// B fragments for two n8 tiles where B[k][n] = s[k][n] (tile stored with k as the row).
template <int LD>
GPT2_DEV void frag_b_kn(const bf16* s, int k0, int n0, uint32_t (&b)[4]) {
  const int l = lane_id();
  const int r = k0 + (l & 7) + 8 * ((l >> 3) & 1);
  const int c = n0 + 8 * (l >> 4);
  ldsm_x4_t(smem_u32(s + r * LD + c), b[0], b[1], b[2], b[3]);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
template <int HD>
__global__ void __launch_bounds__(128) attn_fwd_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ out,
                                                       float* __restrict__ lse, int T, int H, float scale) {
  constexpr int LD = Tile<HD>::LD;
  extern __shared__ __align__(16) uint8_t smem[];
  bf16* Qs = reinterpret_cast<bf16*>(smem);
  bf16* Ks = Qs + BLK * LD;        // two buffers
  bf16* Vs = Ks + 2 * BLK * LD;    // two buffers

  const int nqb = T / BLK;
  const int qb = nqb - 1 - blockIdx.x;  // longest rows first
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int C = H * HD, C3 = 3 * C;
  const bf16* base = qkv + (size_t)b * T * C3 + h * HD;
  const int warp = threadIdx.x >> 5, l = lane_id();
  const float sl2 = scale * kLog2e;

  load_tile<HD>(Qs, base + (size_t)qb * BLK * C3, C3);
  load_tile<HD>(Ks, base + C, C3);
  load_tile<HD>(Vs, base + 2 * C, C3);
  cp_async_commit();

  uint32_t qf[HD / 16][4];
  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int qrow0 = qb * BLK + warp * 16 + (l >> 2);  // this thread's rows: qrow0, qrow0 + 8

  for (int j = 0; j <= qb; ++j) {
    const int buf = j & 1;
    if (j < qb) {
      const int nb = (j + 1) & 1;
      load_tile<HD>(Ks + nb * BLK * LD, base + C + (size_t)(j + 1) * BLK * C3, C3);
      load_tile<HD>(Vs + nb * BLK * LD, base + 2 * C + (size_t)(j + 1) * BLK * C3, C3);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kt = 0; kt < HD / 16; ++kt) frag_a<LD>(Qs, warp * 16, kt * 16, qf[kt]);
    }
    const bf16* Kb = Ks + buf * BLK * LD;
    const bf16* Vb = Vs + buf * BLK * LD;

    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < HD / 16; ++kt) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bb[4];
        frag_b_nk<LD>(Kb, np * 16, kt * 16, bb);
        mma16816(s[2 * np], qf[kt], bb[0], bb[1]);
        mma16816(s[2 * np + 1], qf[kt], bb[2], bb[3]);
      }
    }
    // scale into log2 units, causal mask on the diagonal block, online softmax
    float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[nt][e] * sl2;
        if (j == qb) {
          const int key = j * BLK + nt * 8 + 2 * (l & 3) + (e & 1);
          const int qr = qrow0 + ((e >> 1) << 3);
          if (key > qr) v = -INFINITY;
        }
        s[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      alpha[r] = exp2f(mrow[r] - mx[r]);  // mrow = -inf on the first block -> 0
      mrow[r] = mx[r];
      lrow[r] *= alpha[r];
    }
#pragma unroll
    for (int dt = 0; dt < HD / 8; ++dt) {
      o[dt][0] *= alpha[0]; o[dt][1] *= alpha[0];
      o[dt][2] *= alpha[1]; o[dt][3] *= alpha[1];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = exp2f(s[nt][e] - mrow[e >> 1]);
        s[nt][e] = pv;
        lrow[e >> 1] += pv;
      }
    }
    // O += P V
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      uint32_t a[4];
      a[0] = pack_bf16x2(s[2 * kt][0], s[2 * kt][1]);
      a[1] = pack_bf16x2(s[2 * kt][2], s[2 * kt][3]);
      a[2] = pack_bf16x2(s[2 * kt + 1][0], s[2 * kt + 1][1]);
      a[3] = pack_bf16x2(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
      for (int dp = 0; dp < HD / 16; ++dp) {
        uint32_t bb[4];
        frag_b_kn<LD>(Vb, kt * 16, dp * 16, bb);
        mma16816(o[2 * dp], a, bb[0], bb[1]);
        mma16816(o[2 * dp + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const float inv0 = 1.f / lrow[0], inv1 = 1.f / lrow[1];
  bf16* o0 = out + ((size_t)b * T + qrow0) * C + h * HD;
  bf16* o1 = o0 + (size_t)8 * C;
#pragma unroll
  for (int dt = 0; dt < HD / 8; ++dt) {
    const int c = dt * 8 + 2 * (l & 3);
    *reinterpret_cast<uint32_t*>(o0 + c) = pack_bf16x2(o[dt][0] * inv0, o[dt][1] * inv0);
    *reinterpret_cast<uint32_t*>(o1 + c) = pack_bf16x2(o[dt][2] * inv1, o[dt][3] * inv1);
  }
  if ((l & 3) == 0) {
    float* lp = lse + (size_t)bh * T;
    lp[qrow0] = (mrow[0] + log2f(lrow[0])) * kLn2;
    lp[qrow0 + 8] = (mrow[1] + log2f(lrow[1])) * kLn2;
  }
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------

// D[b,h,t] = sum_d dO[b,t,h,d] * O[b,t,h,d]  (fp32), one thread per (row, head).
template <int HD>
__global__ void attn_bwd_dot_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                    float* __restrict__ Dv, int B, int T, int H) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * T * H) return;
  const int h = idx % H;
  const int row = idx / H;  // b*T + t
  const int C = H * HD;
  const uint4* o = reinterpret_cast<const uint4*>(out + (size_t)row * C + h * HD);
  const uint4* d = reinterpret_cast<const uint4*>(dout + (size_t)row * C + h * HD);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) {
    const uint4 a = o[i], c = d[i];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fa = unpack_bf16x2(aw[k]), fc = unpack_bf16x2(cw[k]);
      acc += fa.x * fc.x + fa.y * fc.y;
    }
  }
  const int b = row / T, t = row % T;
  Dv[((size_t)b * H + h) * T + t] = acc;
}

// Per-warp dQ staging for the bulk reduce: HD/32 boxes of 16 rows x 32 fp32
// (128 bytes per row, 128-byte swizzle), double buffered.
template <int HD>
struct DqStage {
  static constexpr int BOX_BYTES = 16 * 32 * 4;               // 2 KB
  static constexpr int BUF_BYTES = (HD / 32) * BOX_BYTES;     // one iteration of one warp
  static constexpr int BYTES = 4 * 2 * BUF_BYTES;             // 4 warps x 2 buffers
};

template <int HD>
__global__ void __launch_bounds__(128) attn_bwd_kernel(const bf16* __restrict__ qkv, const bf16* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       const float* __restrict__ Dv,
                                                       const __grid_constant__ CUtensorMap tm_dq,
                                                       bf16* __restrict__ dqkv, int T, int H, float scale) {
  constexpr int LD = Tile<HD>::LD;
  constexpr int LDS = BLK + 8;  // dS^T tile [key][query]
  extern __shared__ __align__(1024) uint8_t smem_raw_bwd[];
  // dQ staging first (1024-byte aligned for the swizzle), then the tiles
  uint8_t* smem_al = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw_bwd) + 1023) & ~uintptr_t(1023));
  uint8_t* dq_stage = smem_al;
  uint8_t* smem = smem_al + DqStage<HD>::BYTES;
  bf16* Ks = reinterpret_cast<bf16*>(smem);
  bf16* Vs = Ks + BLK * LD;
  bf16* Qs = Vs + BLK * LD;             // two buffers
  bf16* dOs = Qs + 2 * BLK * LD;        // two buffers
  bf16* dSs = dOs + 2 * BLK * LD;       // [BLK][LDS]
  float* lse_s = reinterpret_cast<float*>(dSs + BLK * LDS);  // two buffers of 64
  float* D_s = lse_s + 2 * BLK;                              // two buffers of 64

  const int nb = T / BLK;
  const int kb = nb - 1 - blockIdx.x;  // fewest query blocks last
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int C = H * HD, C3 = 3 * C;
  const bf16* base = qkv + (size_t)b * T * C3 + h * HD;
  const bf16* dbase = dout + (size_t)b * T * C + h * HD;
  const float* lse_b = lse + (size_t)bh * T;
  const float* D_b = Dv + (size_t)bh * T;
  const int warp = threadIdx.x >> 5, l = lane_id();
  const float sl2 = scale * kLog2e;

  load_tile<HD>(Ks, base + C + (size_t)kb * BLK * C3, C3);
  load_tile<HD>(Vs, base + 2 * C + (size_t)kb * BLK * C3, C3);
  auto load_q = [&](int qi, int buf) {
    load_tile<HD>(Qs + buf * BLK * LD, base + (size_t)qi * BLK * C3, C3);
    load_tile<HD>(dOs + buf * BLK * LD, dbase + (size_t)qi * BLK * C, C);
    if (threadIdx.x < BLK) {
      lse_s[buf * BLK + threadIdx.x] = lse_b[qi * BLK + threadIdx.x] * kLog2e;
      D_s[buf * BLK + threadIdx.x] = D_b[qi * BLK + threadIdx.x];
    }
  };
  load_q(kb, 0);
  cp_async_commit();

  uint32_t kf[HD / 16][4], vf[HD / 16][4];
  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const int key0 = kb * BLK + warp * 16 + (l >> 2);  // this thread's keys: key0, key0 + 8

  for (int qi = kb; qi < nb; ++qi) {
    const int buf = (qi - kb) & 1;
    if (qi + 1 < nb) {
      load_q(qi + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (qi == kb) {
#pragma unroll
      for (int kt = 0; kt < HD / 16; ++kt) {
        frag_a<LD>(Ks, warp * 16, kt * 16, kf[kt]);
        frag_a<LD>(Vs, warp * 16, kt * 16, vf[kt]);
      }
    }
    const bf16* Qb = Qs + buf * BLK * LD;
    const bf16* dOb = dOs + buf * BLK * LD;
    const float* lq = lse_s + buf * BLK;
    const float* Dq = D_s + buf * BLK;

    // S^T = K Q^T and dP^T = V dO^T (16 keys x 64 queries per warp)
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < HD / 16; ++kt) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bb[4];
        frag_b_nk<LD>(Qb, np * 16, kt * 16, bb);
        mma16816(s[2 * np], kf[kt], bb[0], bb[1]);
        mma16816(s[2 * np + 1], kf[kt], bb[2], bb[3]);
        frag_b_nk<LD>(dOb, np * 16, kt * 16, bb);
        mma16816(dp[2 * np], vf[kt], bb[0], bb[1]);
        mma16816(dp[2 * np + 1], vf[kt], bb[2], bb[3]);
      }
    }
    // P^T = exp(S^T * scale - lse[query]); dS^T = P^T * (dP^T - D[query])
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qc = nt * 8 + 2 * (l & 3) + (e & 1);  // query within block
        float pv = exp2f(s[nt][e] * sl2 - lq[qc]);
        if (qi == kb) {
          const int key = key0 + ((e >> 1) << 3);
          if (key > qi * BLK + qc) pv = 0.f;
        }
        s[nt][e] = pv;
        dp[nt][e] = pv * (dp[nt][e] - Dq[qc]);
      }
    }
    // dV += P^T dO ; dK += dS^T Q   (k = query)
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      uint32_t ap[4], ad[4];
      ap[0] = pack_bf16x2(s[2 * kt][0], s[2 * kt][1]);
      ap[1] = pack_bf16x2(s[2 * kt][2], s[2 * kt][3]);
      ap[2] = pack_bf16x2(s[2 * kt + 1][0], s[2 * kt + 1][1]);
      ap[3] = pack_bf16x2(s[2 * kt + 1][2], s[2 * kt + 1][3]);
      ad[0] = pack_bf16x2(dp[2 * kt][0], dp[2 * kt][1]);
      ad[1] = pack_bf16x2(dp[2 * kt][2], dp[2 * kt][3]);
      ad[2] = pack_bf16x2(dp[2 * kt + 1][0], dp[2 * kt + 1][1]);
      ad[3] = pack_bf16x2(dp[2 * kt + 1][2], dp[2 * kt + 1][3]);
#pragma unroll
      for (int dq = 0; dq < HD / 16; ++dq) {
        uint32_t bb[4];
        frag_b_kn<LD>(dOb, kt * 16, dq * 16, bb);
        mma16816(dv[2 * dq], ap, bb[0], bb[1]);
        mma16816(dv[2 * dq + 1], ap, bb[2], bb[3]);
        frag_b_kn<LD>(Qb, kt * 16, dq * 16, bb);
        mma16816(dk[2 * dq], ad, bb[0], bb[1]);
        mma16816(dk[2 * dq + 1], ad, bb[2], bb[3]);
      }
      // stash dS^T (bf16) for the dQ product
      const int r0 = warp * 16 + (l >> 2);
      const int c0 = kt * 16 + 2 * (l & 3);
      *reinterpret_cast<uint32_t*>(dSs + r0 * LDS + c0) = ad[0];
      *reinterpret_cast<uint32_t*>(dSs + (r0 + 8) * LDS + c0) = ad[1];
      *reinterpret_cast<uint32_t*>(dSs + r0 * LDS + c0 + 8) = ad[2];
      *reinterpret_cast<uint32_t*>(dSs + (r0 + 8) * LDS + c0 + 8) = ad[3];
    }
    __syncthreads();
    // dQ[queries of this warp] += scale * dS K   (A = (dS^T)^T from smem, B = K)
    {
      float dqa[HD / 8][4];
#pragma unroll
      for (int i = 0; i < HD / 8; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
        uint32_t a[4];
        frag_a_t<LDS>(dSs, warp * 16, kt * 16, a);
#pragma unroll
        for (int dq = 0; dq < HD / 16; ++dq) {
          uint32_t bb[4];
          frag_b_kn<LD>(Ks, kt * 16, dq * 16, bb);
          mma16816(dqa[2 * dq], a, bb[0], bb[1]);
          mma16816(dqa[2 * dq + 1], a, bb[2], bb[3]);
        }
      }
      // stage scale * dQ (16 x HD fp32) in swizzled shared memory, then one bulk
      // reduce-add per 32-column box into the fp32 accumulator
      uint8_t* buf = dq_stage + (warp * 2 + ((qi - kb) & 1)) * DqStage<HD>::BUF_BYTES;
      if (l == 0) bulk_wait_group_read<1>();  // this buffer's reduce from two iterations ago has read it
      __syncwarp();
      const int r0 = l >> 2;
#pragma unroll
      for (int dt = 0; dt < HD / 8; ++dt) {
        const int c = dt * 8 + 2 * (l & 3);
        const int half = c >> 5, cc = c & 31, j = cc >> 2;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int r = r0 + 8 * rr;
          float2* dst = reinterpret_cast<float2*>(buf + half * DqStage<HD>::BOX_BYTES + r * 128 + ((j ^ (r & 7)) << 4) +
                                                  (cc & 3) * 4);
          *dst = make_float2(dqa[dt][2 * rr] * scale, dqa[dt][2 * rr + 1] * scale);
        }
      }
      fence_async_smem();
      __syncwarp();
      if (l == 0) {
        const int qrow0 = b * T + qi * BLK + warp * 16;
#pragma unroll
        for (int half = 0; half < HD / 32; ++half)
          tma_reduce_add_2d(&tm_dq, smem_u32(buf + half * DqStage<HD>::BOX_BYTES), h * HD + 32 * half, qrow0);
        bulk_commit_group();
      }
    }
    __syncthreads();
  }
  if (l == 0) bulk_wait_group<0>();
  // write dK (scaled) and dV for this warp's 16 keys
  bf16* k0p = dqkv + ((size_t)b * T + key0) * C3 + C + h * HD;
  bf16* v0p = k0p + C;
#pragma unroll
  for (int dt = 0; dt < HD / 8; ++dt) {
    const int c = dt * 8 + 2 * (l & 3);
    *reinterpret_cast<uint32_t*>(k0p + c) = pack_bf16x2(dk[dt][0] * scale, dk[dt][1] * scale);
    *reinterpret_cast<uint32_t*>(k0p + (size_t)8 * C3 + c) = pack_bf16x2(dk[dt][2] * scale, dk[dt][3] * scale);
    *reinterpret_cast<uint32_t*>(v0p + c) = pack_bf16x2(dv[dt][0], dv[dt][1]);
    *reinterpret_cast<uint32_t*>(v0p + (size_t)8 * C3 + c) = pack_bf16x2(dv[dt][2], dv[dt][3]);
  }
}

// dq (fp32 accumulator [B*T, C]) -> the q third of dqkv (bf16); clears the accumulator.
__global__ void attn_dq_convert_kernel(float* __restrict__ dq_acc, bf16* __restrict__ dqkv, int rows, int C) {
  const size_t nvec = (size_t)rows * C / 8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nvec; i += (size_t)gridDim.x * blockDim.x) {
    const size_t e = i * 8;
    const size_t row = e / C, col = e % C;
    float4* src = reinterpret_cast<float4*>(dq_acc + e);
    const float4 a = src[0], c = src[1];
    src[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    src[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<uint4*>(dqkv + row * 3 * C + col) =
        make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
  }
}

template <int HD>
constexpr int fwd_smem() { return 5 * Tile<HD>::BYTES; }
template <int HD>
constexpr int bwd_smem() {
  return 1024 + DqStage<HD>::BYTES + 6 * Tile<HD>::BYTES + BLK * (BLK + 8) * 2 + 4 * BLK * 4;
}

template <int HD>
static cudaError_t fwd(const bf16* qkv, bf16* out, float* lse, int B, int T, int H, cudaStream_t s) {
  static PerDeviceOnce once;
  cudaError_t e = smem_optin(once, attn_fwd_kernel<HD>, fwd_smem<HD>());
  if (e != cudaSuccess) return e;
  dim3 grid(T / BLK, B * H);
  attn_fwd_kernel<HD><<<grid, 128, fwd_smem<HD>(), s>>>(qkv, out, lse, T, H, 1.0f / sqrtf((float)HD));
  return cudaGetLastError();
}

// dq_acc must be all zeros on entry (it is cleared again on exit).
template <int HD>
static cudaError_t bwd(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dv,
                       float* dq_acc, bf16* dqkv, int B, int T, int H, cudaStream_t s) {
  static PerDeviceOnce once;
  cudaError_t e = smem_optin(once, attn_bwd_kernel<HD>, bwd_smem<HD>());
  if (e != cudaSuccess) return e;
  const int rows = B * T * H;
  attn_bwd_dot_kernel<HD><<<(rows + 255) / 256, 256, 0, s>>>(out, dout, Dv, B, T, H);
  const int C = H * HD;
  CUtensorMap tm_dq;
  if (!encode_map_2d(&tm_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dq_acc, C, (uint64_t)B * T, C, 32, 16,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  dim3 grid(T / BLK, B * H);
  attn_bwd_kernel<HD><<<grid, 128, bwd_smem<HD>(), s>>>(qkv, dout, lse, Dv, tm_dq, dqkv, T, H, 1.0f / sqrtf((float)HD));
  const size_t nvec = (size_t)B * T * C / 8;
  int blocks = (int)((nvec + 255) / 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  attn_dq_convert_kernel<<<blocks, 256, 0, s>>>(dq_acc, dqkv, B * T, C);
  return cudaGetLastError();
}

}  // namespace attn
