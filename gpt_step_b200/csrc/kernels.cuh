// Bandwidth-bound kernels of the GPT-2 step: initialisation, embeddings,
// LayerNorm, vocabulary-masked softmax cross-entropy, bias gradients, the
// global gradient norm and the clipped AdamW update.
//
// All of them stream bf16 activations or fp32 state with 16-byte vector loads
// and reduce with warp shuffles; statistics, losses and optimizer math are fp32
// (fp64 for the global sum of squares).
#pragma once
#include "common.cuh"

namespace k {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11) and Box-Muller normals for the
// initialisation ("Pretraining and adapting a language model on a
// dependency-free stack", §4.1: N(0, 0.02), residual projections / sqrt(2L)).
// Counter (c mod 2^32, c div 2^32, kind, 0), key (seed lo, seed hi); each 32-bit
// output x maps to u = ((x >> 9) + 0.5) / 2^23, exact in fp32.
// ---------------------------------------------------------------------------
GPT2_DEV void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
    const uint32_t hi0 = __umulhi(M0, c[0]), lo0 = M0 * c[0];
    const uint32_t hi1 = __umulhi(M1, c[2]), lo1 = M1 * c[2];
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
  }
}

GPT2_DEV float u01(uint32_t x) { return ((float)(x >> 9) + 0.5f) * (1.0f / 8388608.0f); }

// Init one parameter kind: mode 0 = N(0, std) (rows >= zero_row_from are 0),
// 1 = ones, 2 = zeros. Writes the fp32 master and the bf16 copy.
// `ctr_base` is the generator counter of the block's first four elements (its
// element offset within the kind / 4), so that a kind split into per-layer
// blocks draws the same numbers as the kind in one piece; `zero_from` counts
// from the block's start.
__global__ void init_kind_kernel(float* __restrict__ p, bf16* __restrict__ pb, long n, int mode, float stddev,
                                 uint32_t kind, uint64_t seed, long zero_from, long ctr_base) {
  const long nblk = (n + 3) / 4;
  for (long c = blockIdx.x * (long)blockDim.x + threadIdx.x; c < nblk; c += (long)gridDim.x * blockDim.x) {
    float z[4];
    if (mode == 0) {
      const uint64_t cg = (uint64_t)(ctr_base + c);
      uint32_t ctr[4] = {(uint32_t)(cg & 0xFFFFFFFFu), (uint32_t)(cg >> 32), kind, 0u};
      philox4x32_10(ctr, (uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32));
      const float r01 = sqrtf(-2.0f * logf(u01(ctr[0])));
      const float r23 = sqrtf(-2.0f * logf(u01(ctr[2])));
      float s1, c1, s3, c3;
      sincospif(2.0f * u01(ctr[1]), &s1, &c1);
      sincospif(2.0f * u01(ctr[3]), &s3, &c3);
      z[0] = r01 * c1; z[1] = r01 * s1; z[2] = r23 * c3; z[3] = r23 * s3;
#pragma unroll
      for (int j = 0; j < 4; ++j) z[j] *= stddev;
    } else {
      const float v = mode == 1 ? 1.0f : 0.0f;
      z[0] = z[1] = z[2] = z[3] = v;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long e = 4 * c + j;
      if (e < n) {
        const float v = (e >= zero_from) ? 0.0f : z[j];
        p[e] = v;
        pb[e] = __float2bfloat16_rn(v);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a1  embedding: x[n, :] = wte[tok[n], :] + wpe[n % T, :]   (bf16 copies)
// ---------------------------------------------------------------------------
__global__ void embed_fwd_kernel(const int32_t* __restrict__ tok, const bf16* __restrict__ wte,
                                 const bf16* __restrict__ wpe, bf16* __restrict__ x, int N, int T, int C, int V,
                                 int* err) {
  pdl_begin();
  const int vpr = C / 8;
  const long total = (long)N * vpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int n = (int)(i / vpr), c = (int)(i % vpr) * 8;
    int t = tok[n];
    if (t < 0 || t >= V) {
      if (c == 0) atomicOr(err, DEVERR_TOKEN_RANGE);
      t = 0;
    }
    const uint4 a = *reinterpret_cast<const uint4*>(wte + (size_t)t * C + c);
    const uint4 b = *reinterpret_cast<const uint4*>(wpe + (size_t)(n % T) * C + c);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fa = unpack_bf16x2(aw[j]), fb = unpack_bf16x2(bw[j]);
      o[j] = pack_bf16x2(fa.x + fb.x, fa.y + fb.y);
    }
    *reinterpret_cast<uint4*>(x + (size_t)n * C + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// a1 backward, position part: dwpe[t, :] += sum_b dx[b, t, :]   (deterministic)
__global__ void embed_bwd_wpe_kernel(const bf16* __restrict__ dx, float* __restrict__ dwpe, int B, int T, int C) {
  pdl_begin();
  const int vpr = C / 8;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * vpr) return;
  const int t = i / vpr, c = (i % vpr) * 8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int b = 0; b < B; ++b) {
    const uint4 u = *reinterpret_cast<const uint4*>(dx + ((size_t)b * T + t) * C + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16x2(w[j]);
      acc[2 * j] += f.x;
      acc[2 * j + 1] += f.y;
    }
  }
  float4* d = reinterpret_cast<float4*>(dwpe + (size_t)t * C + c);
  float4 d0 = d[0], d1 = d[1];
  d0.x += acc[0]; d0.y += acc[1]; d0.z += acc[2]; d0.w += acc[3];
  d1.x += acc[4]; d1.y += acc[5]; d1.z += acc[6]; d1.w += acc[7];
  d[0] = d0;
  d[1] = d1;
}

// a1 backward, token part: dwte[tok[n], :] += dx[n, :]. A CTA takes kEmbRows
// consecutive positions; rows with the same token id are summed inside the CTA
// (in position order) and added into dwte once per id by fp32 vector atomics, so
// a frequent id (the Zipf head of the stream) sees one atomic per CTA instead
// of one per occurrence.
constexpr int kEmbRows = 64;
__global__ void __launch_bounds__(256) embed_bwd_wte_kernel(const int32_t* __restrict__ tok,
                                                            const bf16* __restrict__ dx, float* __restrict__ dwte,
                                                            int N, int C, int V) {
  pdl_begin();
  __shared__ int st[kEmbRows];
  __shared__ unsigned char lead[kEmbRows];
  const int r0 = blockIdx.x * kEmbRows;
  if (threadIdx.x < kEmbRows) {
    const int n = r0 + threadIdx.x;
    const int t = n < N ? tok[n] : -1;
    st[threadIdx.x] = (t >= 0 && t < V) ? t : -1;
  }
  __syncthreads();
  if (threadIdx.x < kEmbRows) {
    const int t = st[threadIdx.x];
    bool first = t >= 0;
    for (int j = 0; j < (int)threadIdx.x && first; ++j) first = st[j] != t;
    lead[threadIdx.x] = first ? 1 : 0;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int vpr = C / 8;
  // leaders in round robin over the warps; a lane owns the 16-byte chunks lane, lane + 32, ..
  int k = 0;
  for (int i = 0; i < kEmbRows; ++i) {
    if (!lead[i]) continue;
    if ((k++ % nw) != warp) continue;
    const int t = st[i];
    for (int v = lane; v < vpr; v += 32) {
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int j = i; j < kEmbRows; ++j) {
        if (st[j] != t) continue;
        const uint4 u = *reinterpret_cast<const uint4*>(dx + (size_t)(r0 + j) * C + v * 8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = unpack_bf16x2(w[q]);
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      }
      float* d = dwte + (size_t)t * C + v * 8;
      red_add_f32x4(d, acc[0], acc[1], acc[2], acc[3]);
      red_add_f32x4(d + 4, acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// ---------------------------------------------------------------------------
// a2/a6/a9  LayerNorm forward: a warp normalises RP rows at a time (RP = 2 for
// C <= 768, else 1) in a grid-stride loop over the rows, the next RP rows'
// loads in flight while these are normalised; the RP rows' warp reductions
// are interleaved, so their shuffle latencies overlap (the grid is the
// resident-CTA count, so there is no partial last wave). fp32 statistics (eps
// 1e-5, biased variance), y = (x - mean) * rstd * w + b in bf16.
// ---------------------------------------------------------------------------
constexpr int kLnFwdWarps = 8;   // warps per CTA
__host__ __device__ constexpr int ln_fwd_rows(int C) { return C <= 768 ? 2 : 1; }
// CTAs per SM: as many as the rows' registers allow without spilling
__host__ __device__ constexpr int ln_fwd_minb(int C) { return C <= 768 ? 2 : (C <= 1024 ? 3 : 2); }
template <int C>
__global__ void __launch_bounds__(kLnFwdWarps * 32, ln_fwd_minb(C)) layernorm_fwd_kernel(const bf16* __restrict__ x,
                                                                        const float* __restrict__ w,
                                                                        const float* __restrict__ b,
                                                                        bf16* __restrict__ y, float* __restrict__ mean,
                                                                        float* __restrict__ rstd, int rows) {
  pdl_begin();
  constexpr int NV = C / 8;                 // 16-byte vectors per row
  constexpr int VPL = (NV + 31) / 32;       // vectors per lane
  constexpr int RP = ln_fwd_rows(C);        // rows a warp normalises together
  const int l = lane_id();
  const int stride = gridDim.x * kLnFwdWarps * RP;
  int row = (blockIdx.x * kLnFwdWarps + (threadIdx.x >> 5)) * RP;
  auto load = [&](int r, uint4 (&u)[RP][VPL]) {
#pragma unroll
    for (int p = 0; p < RP; ++p)
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int vi = l + 32 * i;
        u[p][i] = (vi < NV && r + p < rows) ? __ldcs(reinterpret_cast<const uint4*>(x + (size_t)(r + p) * C) + vi)
                                            : make_uint4(0u, 0u, 0u, 0u);
      }
  };
  uint4 cur[RP][VPL], nxt[RP][VPL];
  load(row, cur);
  for (; row < rows; row += stride) {
    load(row + stride, nxt);
    float v[RP][VPL][8];
    float s[RP];
#pragma unroll
    for (int p = 0; p < RP; ++p) {
      s[p] = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const uint32_t wv[4] = {cur[p][i].x, cur[p][i].y, cur[p][i].z, cur[p][i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(wv[j]);
          v[p][i][2 * j] = f.x;
          v[p][i][2 * j + 1] = f.y;
          s[p] += f.x + f.y;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int p = 0; p < RP; ++p) s[p] += __shfl_xor_sync(0xffffffffu, s[p], o);
    float mu[RP], ss[RP];
#pragma unroll
    for (int p = 0; p < RP; ++p) {
      mu[p] = s[p] * (1.0f / C);
      ss[p] = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (l + 32 * i < NV)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float d = v[p][i][j] - mu[p];
            ss[p] += d * d;
          }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int p = 0; p < RP; ++p) ss[p] += __shfl_xor_sync(0xffffffffu, ss[p], o);
    float rs[RP];
#pragma unroll
    for (int p = 0; p < RP; ++p) rs[p] = rsqrtf(ss[p] * (1.0f / C) + 1e-5f);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = l + 32 * i;
      if (vi < NV) {
        // gain and shift: L1-resident after the first row
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(w + vi * 8));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(w + vi * 8 + 4));
        const float4 b0 = __ldg(reinterpret_cast<const float4*>(b + vi * 8));
        const float4 b1 = __ldg(reinterpret_cast<const float4*>(b + vi * 8 + 4));
        const float ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int p = 0; p < RP; ++p) {
          if (row + p >= rows) continue;
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            o[j] = pack_bf16x2((v[p][i][2 * j] - mu[p]) * rs[p] * ww[2 * j] + bb[2 * j],
                               (v[p][i][2 * j + 1] - mu[p]) * rs[p] * ww[2 * j + 1] + bb[2 * j + 1]);
          // a plain store: the next GEMM reads y while it is still in L2
          *reinterpret_cast<uint4*>(y + (size_t)(row + p) * C + vi * 8) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    // lane p writes the statistics of row p
#pragma unroll
    for (int p = 0; p < RP; ++p)
      if (l == p && row + p < rows) {
        mean[row + p] = mu[p];
        rstd[row + p] = rs[p];
      }
#pragma unroll
    for (int p = 0; p < RP; ++p)
#pragma unroll
      for (int i = 0; i < VPL; ++i) cur[p][i] = nxt[p][i];
  }
}

// LayerNorm backward: dx = rstd * (dy*w - mean(dy*w) - xhat * mean(dy*w*xhat))
// (+ dresid, the gradient flowing along the residual stream), written in bf16.
// One warp per row, rows in a grid-stride loop; a lane always owns the same
// columns (16-byte chunk vi = lane + 32 i), so its column sums of dy*xhat, dy
// and (optionally) of its output dx stay in registers across rows (C <= 1024;
// wider rows keep them in warp-private shared memory). At the end the warps'
// sums are combined in a fixed order and the CTA writes one partial row per
// quantity to `part` ([grid][NQ][C], NQ = 3 with the dx sum, else 2), summed in
// a fixed order afterwards. The dx column sum is the gradient of the bias of
// the projection that wrote the residual stream (its output gradient is dx).
// Warps per CTA and CTAs per SM by row width: enough rows in flight per SM
// for the HBM latency, with the register column sums unspilled.
__host__ __device__ constexpr int ln_bwd_warps(int C) { return C <= 512 ? 8 : (C == 768 ? 12 : (C == 1024 ? 8 : 4)); }
__host__ __device__ constexpr int ln_bwd_minb(int C) { return (C <= 512 || C > 1024) ? 2 : 1; }
template <int C>
struct LnBwdCfg {
  static constexpr int WARPS = ln_bwd_warps(C);
  static constexpr int MINB = ln_bwd_minb(C);
  static constexpr int SMEM = WARPS * 3 * C * 4;
};

template <int C>
__global__ void __launch_bounds__(LnBwdCfg<C>::WARPS * 32, LnBwdCfg<C>::MINB)
    layernorm_bwd_kernel(const bf16* __restrict__ dy, const bf16* __restrict__ x, const float* __restrict__ mean,
                         const float* __restrict__ rstd, const float* __restrict__ w, const bf16* dresid, bf16* dx,
                         float* __restrict__ part, int rows, int with_dxsum, float* dw, float* db, float* dbias) {
  pdl_begin();
  constexpr int NV = C / 8;
  constexpr int VPL = (NV + 31) / 32;
  constexpr int WARPS = LnBwdCfg<C>::WARPS;
  constexpr bool kRegAcc = VPL <= 4;
  extern __shared__ __align__(16) float ln_acc[];  // [WARPS][3][C]
  const int warp = threadIdx.x >> 5, l = lane_id();
  float* acc = ln_acc + warp * 3 * C;
  float ra[kRegAcc ? VPL : 1][3][8];
#pragma unroll
  for (int i = 0; i < (kRegAcc ? VPL : 1); ++i)
#pragma unroll
    for (int q = 0; q < 3; ++q)
#pragma unroll
      for (int j = 0; j < 8; ++j) ra[i][q][j] = 0.f;
  if (!kRegAcc) {
    for (int i = l; i < 3 * C; i += 32) acc[i] = 0.f;
    __syncwarp();
  }
  const int nq = with_dxsum ? 3 : 2;
  // the weights of this lane's columns, loaded once
  float wv[VPL][8];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = l + 32 * i;
    if (vi < NV) {
      const float4 w0 = __ldg(reinterpret_cast<const float4*>(w + vi * 8));
      const float4 w1 = __ldg(reinterpret_cast<const float4*>(w + vi * 8 + 4));
      wv[i][0] = w0.x; wv[i][1] = w0.y; wv[i][2] = w0.z; wv[i][3] = w0.w;
      wv[i][4] = w1.x; wv[i][5] = w1.y; wv[i][6] = w1.z; wv[i][7] = w1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[i][j] = 0.f;
    }
  }
  for (int row = blockIdx.x * WARPS + warp; row < rows; row += gridDim.x * WARPS) {
    const float mu = mean[row], rs = rstd[row];
    uint4 ux[VPL], ud[VPL], ur[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = l + 32 * i;
      ur[i] = make_uint4(0u, 0u, 0u, 0u);
      if (vi < NV) {
        ux[i] = __ldcs(reinterpret_cast<const uint4*>(x + (size_t)row * C + vi * 8));
        ud[i] = __ldcs(reinterpret_cast<const uint4*>(dy + (size_t)row * C + vi * 8));
        if (dresid != nullptr) ur[i] = __ldcs(reinterpret_cast<const uint4*>(dresid + (size_t)row * C + vi * 8));
      }
    }
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = l + 32 * i;
      if (vi < NV) {
        const uint32_t xw[4] = {ux[i].x, ux[i].y, ux[i].z, ux[i].w}, dw4[4] = {ud[i].x, ud[i].y, ud[i].z, ud[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 fx = unpack_bf16x2(xw[j]), fd = unpack_bf16x2(dw4[j]);
          const float xh0 = (fx.x - mu) * rs, xh1 = (fx.y - mu) * rs;
          if (kRegAcc) {
            ra[i][0][2 * j] += fd.x * xh0;
            ra[i][0][2 * j + 1] += fd.y * xh1;
            ra[i][1][2 * j] += fd.x;
            ra[i][1][2 * j + 1] += fd.y;
          } else {
            float* a0 = acc + vi * 8;
            float* a1 = acc + C + vi * 8;
            a0[2 * j] += fd.x * xh0;
            a0[2 * j + 1] += fd.y * xh1;
            a1[2 * j] += fd.x;
            a1[2 * j + 1] += fd.y;
          }
          const float g0 = fd.x * wv[i][2 * j], g1 = fd.y * wv[i][2 * j + 1];
          s1 += g0 + g1;
          s2 += g0 * xh0 + g1 * xh1;
        }
      }
    }
    const float m1 = warp_sum(s1) * (1.0f / C), m2 = warp_sum(s2) * (1.0f / C);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = l + 32 * i;
      if (vi < NV) {
        const uint32_t xw[4] = {ux[i].x, ux[i].y, ux[i].z, ux[i].w}, dw4[4] = {ud[i].x, ud[i].y, ud[i].z, ud[i].w};
        const uint32_t rw[4] = {ur[i].x, ur[i].y, ur[i].z, ur[i].w};
        float r[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 fx = unpack_bf16x2(xw[j]), fd = unpack_bf16x2(dw4[j]), fr = unpack_bf16x2(rw[j]);
          r[2 * j] = (fd.x * wv[i][2 * j] - m1 - (fx.x - mu) * rs * m2) * rs + fr.x;
          r[2 * j + 1] = (fd.y * wv[i][2 * j + 1] - m1 - (fx.y - mu) * rs * m2) * rs + fr.y;
        }
        const uint4 o = make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                                   pack_bf16x2(r[6], r[7]));
        *reinterpret_cast<uint4*>(dx + (size_t)row * C + vi * 8) = o;
        if (with_dxsum) {
          // the bias gradient sees the stored (bf16) residual gradient
          const uint32_t ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = unpack_bf16x2(ow[j]);
            if (kRegAcc) {
              ra[i][2][2 * j] += f.x;
              ra[i][2][2 * j + 1] += f.y;
            } else {
              float* a2 = acc + 2 * C + vi * 8;
              a2[2 * j] += f.x;
              a2[2 * j + 1] += f.y;
            }
          }
        }
      }
    }
  }
  if (kRegAcc) {
#pragma unroll
    for (int i = 0; i < (kRegAcc ? VPL : 1); ++i) {
      const int vi = l + 32 * i;
      if (vi < NV) {
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          float4* dst = reinterpret_cast<float4*>(acc + q * C + vi * 8);
          dst[0] = make_float4(ra[i][q][0], ra[i][q][1], ra[i][q][2], ra[i][q][3]);
          dst[1] = make_float4(ra[i][q][4], ra[i][q][5], ra[i][q][6], ra[i][q][7]);
        }
      }
    }
  }
  __syncthreads();
  if (part != nullptr) {
    // combine the warps' column sums in a fixed order (deterministic); a second
    // launch sums the CTAs' partial rows
    for (int c = threadIdx.x; c < nq * C; c += WARPS * 32) {
      float sum = 0.f;
#pragma unroll
      for (int wi = 0; wi < WARPS; ++wi) sum += ln_acc[wi * 3 * C + c];
      part[(size_t)blockIdx.x * nq * C + c] = sum;
    }
  } else {
    // the CTA's column sums go straight into dw, db (and dbias) by vector atomics:
    // one launch, summation order across CTAs unspecified
    for (int c = 4 * threadIdx.x; c < nq * C; c += 4 * WARPS * 32) {
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int wi = 0; wi < WARPS; ++wi) {
        const float4 a = *reinterpret_cast<const float4*>(ln_acc + wi * 3 * C + c);
        sum.x += a.x; sum.y += a.y; sum.z += a.z; sum.w += a.w;
      }
      float* dst = c < C ? dw + c : (c < 2 * C ? db + (c - C) : dbias + (c - 2 * C));
      red_add_f32x4(dst, sum.x, sum.y, sum.z, sum.w);
    }
  }
}

// Sum the nblk partial rows of `part` ([nblk][width], width = nq * C) column by
// column in a fixed order and add them into out0 (dw), out1 (db) and out2 (bias
// grad, when nq == 3). Block (32 x 8): 32 columns, 8 row-lanes, then a fold.
__global__ void __launch_bounds__(256) partial_rows_reduce_kernel(const float* __restrict__ part, int nblk, int width,
                                                                 float* out0, float* out1, float* out2, int C) {
  pdl_begin();
  __shared__ float red[8][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + tx;
  float s = 0.f;
  if (col < width)
    for (int i = ty; i < nblk; i += 8) s += part[(size_t)i * width + col];
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && col < width) {
#pragma unroll
    for (int y = 1; y < 8; ++y) s += red[y][tx];
    const int which = col / C, c = col % C;
    float* dst = which == 0 ? out0 : (which == 1 ? out1 : out2);
    dst[c] += s;
  }
}

// ---------------------------------------------------------------------------
// bias gradient: db[n] += sum_m dout[m, n] (bf16 input, two deterministic passes)
// Pass 1: block (32 x 8 threads) covers 256 columns over a strip of rows.
// ---------------------------------------------------------------------------
// With part == nullptr the strip's sums are added into db directly (fp32 atomics,
// no second pass).
__global__ void __launch_bounds__(256) colsum_partial_kernel(const bf16* __restrict__ a, float* __restrict__ part,
                                                             int M, int N, int rows_per_strip, float* db) {
  pdl_begin();
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c = (blockIdx.x * 32 + tx) * 8;
  const int r0 = blockIdx.y * rows_per_strip;
  const int r1 = min(M, r0 + rows_per_strip);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (c < N) {
    int r = r0 + ty;
    // eight independent rows per iteration keep eight 16-byte loads in flight
    for (; r + 56 < r1; r += 64) {
      uint4 u[8];
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) u[k2] = __ldcs(reinterpret_cast<const uint4*>(a + (size_t)(r + 8 * k2) * N + c));
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) {
        const uint32_t w[4] = {u[k2].x, u[k2].y, u[k2].z, u[k2].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(w[j]);
          acc[2 * j] += f.x;
          acc[2 * j + 1] += f.y;
        }
      }
    }
    for (; r < r1; r += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(a + (size_t)r * N + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(w[j]);
        acc[2 * j] += f.x;
        acc[2 * j + 1] += f.y;
      }
    }
  }

  __shared__ float red[8][32][9];
#pragma unroll
  for (int j = 0; j < 8; ++j) red[ty][tx][j] = acc[j];
  __syncthreads();
  if (ty == 0 && c < N) {
    float s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      s[j] = 0.f;
#pragma unroll
      for (int y = 0; y < 8; ++y) s[j] += red[y][tx][j];
    }
    if (part != nullptr) {
#pragma unroll
      for (int j = 0; j < 8; ++j) part[(size_t)blockIdx.y * N + c + j] = s[j];
    } else {
      red_add_f32x4(db + c, s[0], s[1], s[2], s[3]);
      red_add_f32x4(db + c + 4, s[4], s[5], s[6], s[7]);
    }
  }
}

__global__ void colsum_final_kernel(const float* __restrict__ part, float* __restrict__ db, int strips, int N) {
  pdl_begin();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N) return;
  float s = 0.f;
  for (int i = 0; i < strips; ++i) s += part[(size_t)i * N + c];
  db[c] += s;
}

// ---------------------------------------------------------------------------
// a11  vocabulary-masked softmax cross-entropy, forward and backward fused.
// One CTA per row: the bf16 logits row is read once into shared memory while a
// running (max, sum of exp) is kept over the REAL columns j < V only; the row is
// then overwritten in place with dz = (softmax_j - [j == target]) * dscale for
// j < V and exactly 0 for the padded columns j >= V ("Pretraining and adapting
// a language model on a dependency-free stack", §4.1). loss = lse - z[target].
// ---------------------------------------------------------------------------
constexpr float kLog2eF = 1.4426950408889634f, kLn2F = 0.6931471805599453f;
constexpr int kCeThreads = 256;
constexpr int kCeUnroll = 4;

// Base-2 online softmax: logits are scaled by log2(e) once (y = z * log2e), so
// every exponential is one ex2 of an FFMA. Only the row's last 8-wide chunks can
// hold padded ids (>= V); full chunks skip the per-element column test.
GPT2_DEV void bf16x8_to_f32(uint4 u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// Online (max, sum of 2^(y - max)) over the real columns of one chunk, in log2 units.
GPT2_DEV void ce_accumulate(uint4 u, int col0, int V, float& m, float& s) {
  float f[8];
  bf16x8_to_f32(u, f);
  const bool full = col0 + 8 <= V;
  float lm = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    f[j] *= kLog2eF;
    if (full || col0 + j < V) lm = fmaxf(lm, f[j]);
  }
  if (lm == -INFINITY) return;
  if (lm > m) {
    s *= ex2_approx(m - lm);
    m = lm;
  }
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (full || col0 + j < V) acc += ex2_approx(f[j] - m);
  s += acc;
}

GPT2_DEV void ce_combine(float& m, float& s, float om, float os) {
  const float nm = fmaxf(m, om);
  s = (nm == -INFINITY) ? 0.f : s * ex2_approx(m - nm) + os * ex2_approx(om - nm);
  m = nm;
}

// One CTA per row, no shared-memory staging (rows whose target equals
// ignore_index, when one is given, get loss 0 and a zero gradient): pass 1 streams the bf16 row
// (kCeUnroll 16-byte loads in flight per thread) for the running (max, sum of
// exp) over the real columns; pass 2 reads the row again (from L2) and
// overwrites it with dz. With `part` given, pass 1 instead combines the row's
// `slots` (max, sum) partials that the logits GEMM's epilogue left (the same
// base-2 quantities over the same stored values), and the row is read once.
// With `tgt_val` given as well (a loss without gradient), the target logit is
// taken from tgt_val[row] and the logits are not read at all (may be null);
// tgt_val may alias `losses`.
__global__ void __launch_bounds__(kCeThreads) softmax_ce_kernel(bf16* __restrict__ logits,
                                                                const int32_t* __restrict__ targets,
                                                                float* __restrict__ losses, int V, int Vp,
                                                                float dscale, int write_grad, int* err,
                                                                int ignore_index, const float2* __restrict__ part,
                                                                int slots, const float* tgt_val) {
  pdl_begin();
  __shared__ float red_m[kCeThreads / 32], red_s[kCeThreads / 32];
  __shared__ float bc[2];
  const int row = blockIdx.x;
  uint4* zr = reinterpret_cast<uint4*>(logits + (size_t)row * Vp);
  const int nv = Vp / 8;
  if (targets[row] == ignore_index) {
    // an ignored position: loss 0, gradient exactly 0, not an error
    if (threadIdx.x == 0) losses[row] = 0.f;
    if (write_grad)
      for (int i = threadIdx.x; i < nv; i += kCeThreads) __stcs(zr + i, make_uint4(0u, 0u, 0u, 0u));
    return;
  }
  float m = -INFINITY, s = 0.f;
  if (part != nullptr) {
    const float2* pr = part + (size_t)row * slots;
    for (int i = threadIdx.x; i < slots; i += kCeThreads) {
      const float2 v = __ldcs(pr + i);
      ce_combine(m, s, v.x, v.y);
    }
  } else {
    for (int i0 = threadIdx.x; i0 < nv; i0 += kCeThreads * kCeUnroll) {
      uint4 u[kCeUnroll];
#pragma unroll
      for (int k2 = 0; k2 < kCeUnroll; ++k2) {
        const int i = i0 + k2 * kCeThreads;
        u[k2] = i < nv ? __ldcg(zr + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k2 = 0; k2 < kCeUnroll; ++k2) {
        const int i = i0 + k2 * kCeThreads;
        if (i < nv) ce_accumulate(u[k2], i * 8, V, m, s);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    ce_combine(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
  const int warp = threadIdx.x >> 5, l = lane_id();
  if (l == 0) { red_m[warp] = m; red_s[warp] = s; }
  __syncthreads();
  if (warp == 0) {
    m = l < kCeThreads / 32 ? red_m[l] : -INFINITY;
    s = l < kCeThreads / 32 ? red_s[l] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      ce_combine(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
    if (l == 0) { bc[0] = m; bc[1] = s; }
  }
  __syncthreads();
  const float M2 = bc[0];                      // row max in log2 units
  const float S2 = bc[1];                      // sum of 2^(y - M2)
  int t = targets[row];
  const bool tok_ok = (t >= 0 && t < V);
  if (!tok_ok) {
    if (threadIdx.x == 0) atomicOr(err, DEVERR_TOKEN_RANGE);
    t = -1;
  }
  if (threadIdx.x == 0) {
    // loss = lse - z[t] = (M2 + log2 S2) * ln2 - z[t]
    const float zt = !tok_ok ? 0.f : (tgt_val ? tgt_val[row] : __bfloat162float(logits[(size_t)row * Vp + t]));
    losses[row] = tok_ok ? ((M2 + log2f(S2)) * kLn2F - zt) : 0.f;
  }
  if (!write_grad) return;
  __syncthreads();  // the target logit is read before the row is overwritten
  const float g = dscale / S2;                 // dz = (2^(y - M2) / S2 - [col == t]) * dscale
  for (int i0 = threadIdx.x; i0 < nv; i0 += kCeThreads * kCeUnroll) {
    uint4 u[kCeUnroll];
#pragma unroll
    for (int k2 = 0; k2 < kCeUnroll; ++k2) {
      const int i = i0 + k2 * kCeThreads;
      u[k2] = i < nv ? __ldcg(zr + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k2 = 0; k2 < kCeUnroll; ++k2) {
      const int i = i0 + k2 * kCeThreads;
      if (i >= nv) continue;
      const int c0 = i * 8;
      float f[8];
      bf16x8_to_f32(u[k2], f);
      float gv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) gv[j] = ex2_approx(fmaf(f[j], kLog2eF, -M2)) * g;
      if (c0 + 8 > V) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (c0 + j >= V) gv[j] = 0.f;       // padded ids: exactly zero gradient
      }
      if ((unsigned)(t - c0) < 8u) gv[t - c0] -= dscale;
      __stcs(zr + i, make_uint4(pack_bf16x2(gv[0], gv[1]), pack_bf16x2(gv[2], gv[3]), pack_bf16x2(gv[4], gv[5]),
                                pack_bf16x2(gv[6], gv[7])));
    }
  }
}

// Sum n per-row losses (fp64 accumulation) into acc[0] and store the micro-batch
// mean in *mean_out.
__global__ void loss_reduce_kernel(const float* __restrict__ losses, int n, double* __restrict__ acc,
                                   float* __restrict__ mean_out) {
  pdl_begin();
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += (double)losses[i];
  s = warp_sum_d(s);
  if (lane_id() == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    s = warp_sum_d(s);
    if (threadIdx.x == 0) {
      acc[0] += s;
      *mean_out = (float)(s / n);
    }
  }
}

// ---------------------------------------------------------------------------
// a12  global gradient norm. Pass 1: per-block fp64 partial sums of g^2 over
// the flat fp32 gradient array (float4 loads).
// ---------------------------------------------------------------------------
// Half-open ranges of float4 indices into the flat parameter arrays (passed by value).
struct Ranges4 {
  static constexpr int kMax = 64;
  long begin[kMax], end[kMax];
  int n;
};

// Partial sums of squares of g over the ranges, one per block.
__global__ void __launch_bounds__(512) sumsq_partial_kernel(const float* __restrict__ g, const Ranges4 rg,
                                                            double* __restrict__ part) {
  pdl_begin();
  __shared__ double red[16];
  double s = 0.0;
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const long stride = (long)gridDim.x * blockDim.x;
  for (int r = 0; r < rg.n; ++r) {
    long i = rg.begin[r] + blockIdx.x * (long)blockDim.x + threadIdx.x;
    // four loads in flight per thread
    for (; i + 3 * stride < rg.end[r]; i += 4 * stride) {
      float4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = __ldcs(g4 + i + q * stride);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        s += (double)v[q].x * v[q].x + (double)v[q].y * v[q].y + (double)v[q].z * v[q].z + (double)v[q].w * v[q].w;
    }
    for (; i < rg.end[r]; i += stride) {
      const float4 v = g4[i];
      s += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
    }
  }
  s = warp_sum_d(s);
  if (lane_id() == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = threadIdx.x < 16 ? red[threadIdx.x] : 0.0;
    s = warp_sum_d(s);
    if (threadIdx.x == 0) part[blockIdx.x] = s;
  }
}

// Optimizer scalars shared by the norm and AdamW kernels (device memory).
struct StepScalars {
  double loss_sum;      // sum of micro-batch losses x rows since the last step
  float norm;           // pre-clip norm of g / n_micro
  float gscale;         // multiplier applied to raw g: min(1, clip/norm) / n_micro
  int skip;             // 1: non-finite loss or norm, update not applied
  int n_micro;          // micro-steps accumulated (device copy)
  float last_loss;      // mean loss of the last completed step
  float last_norm;      // pre-clip norm of the last completed step
  float micro_loss;     // mean loss of the last micro-batch
  int pad;
};

// Pass 2: combine partials; derive the clip multiplier; flag non-finite steps.
__global__ void norm_finalize_kernel(const double* __restrict__ part, int nparts, StepScalars* sc, int n_micro,
                                     long rows_per_micro, float clip, int* err) {
  pdl_begin();
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) s += part[i];
  s = warp_sum_d(s);
  if (lane_id() == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    const double norm = sqrt(t) / (double)n_micro;
    const double mean_loss = sc->loss_sum / ((double)rows_per_micro * n_micro);
    const bool finite = isfinite(norm) && isfinite(mean_loss);
    const double k = (norm > clip) ? (double)clip / norm : 1.0;
    sc->norm = (float)norm;
    sc->gscale = (float)(k / (double)n_micro);
    sc->skip = finite ? 0 : 1;
    sc->last_loss = (float)mean_loss;
    sc->last_norm = (float)norm;
    sc->loss_sum = 0.0;
    if (!finite) atomicOr(err, DEVERR_NONFINITE);
  }
}

// Sum of the partials into one double (the caller's device value).
__global__ void sum_partials_kernel(const double* __restrict__ part, int nparts, double* __restrict__ out) {
  pdl_begin();
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) s += part[i];
  s = warp_sum_d(s);
  if (lane_id() == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    *out = t;
  }
}

// ---------------------------------------------------------------------------
// a13  clipped AdamW over the given float4 ranges of the flat parameter arrays.
// The 2-D weights (which take decoupled weight decay) are exactly the elements
// from decay_from4 * 4 on; the zero padding there stays zero. Writes p, m, v,
// the bf16 copy and clears g in the ranges. If the step is flagged non-finite
// only g is cleared.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    bf16* __restrict__ pb, const Ranges4 rg, long decay_from4,
                                                    const StepScalars* __restrict__ sc, float lr, float beta1,
                                                    float beta2, float eps, float wd, float bc1, float bc2) {
  pdl_begin();
  const float gs = sc->gscale;
  const int skip = sc->skip;
  for (int r = 0; r < rg.n; ++r)
  for (long i = rg.begin[r] + blockIdx.x * (long)blockDim.x + threadIdx.x; i < rg.end[r];
       i += (long)gridDim.x * blockDim.x) {
    const long e = i * 4;
    float4* g4 = reinterpret_cast<float4*>(g) + i;
    if (skip) {
      *g4 = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const float lam = i >= decay_from4 ? wd : 0.f;
    float4 gv = *g4;
    float4 pv = reinterpret_cast<float4*>(p)[i];
    float4 mv = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    float* gp = &gv.x;
    float* pp = &pv.x;
    float* mp = &mv.x;
    float* vp = &vv.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float gg = gp[j] * gs;
      mp[j] = beta1 * mp[j] + (1.0f - beta1) * gg;
      vp[j] = beta2 * vp[j] + (1.0f - beta2) * gg * gg;
      const float mh = mp[j] / bc1;
      const float vh = vp[j] / bc2;
      pp[j] = pp[j] - lr * (mh / (sqrtf(vh) + eps) + lam * pp[j]);
    }
    reinterpret_cast<float4*>(p)[i] = pv;
    reinterpret_cast<float4*>(m)[i] = mv;
    reinterpret_cast<float4*>(v)[i] = vv;
    *g4 = make_float4(0.f, 0.f, 0.f, 0.f);
    uint2 pk;
    pk.x = pack_bf16x2(pv.x, pv.y);
    pk.y = pack_bf16x2(pv.z, pv.w);
    *reinterpret_cast<uint2*>(pb + e) = pk;
  }
}

// fp32 -> bf16 copy (used after host writes of parameters).
__global__ void to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, long n) {
  pdl_begin();
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// Bounded-wait self-test: lane 0 waits on a barrier whose phase nothing
// completes (its count is 1 and nobody arrives); the wait gives up after
// limit_ns, records DEVERR_TIMEOUT in err and the kernel returns normally.
__global__ void wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_limit(smem_u32(&bar), 0, err, limit_ns);
  __syncwarp();
}

}  // namespace k
