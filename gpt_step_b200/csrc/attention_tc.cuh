// Causal flash attention forward on the 5th-generation tensor cores (head size 64 or 32).
//
// Same operation as attn::attn_fwd_kernel (grow_a_language_model_intro,
// activities 5-6: softmax(Q K^T / sqrt(d)) V with a causal mask, per head),
// organised for tcgen05:
//
//   CTA     persistent, two an SM; a tile is one (batch, head) and 128 query
//           rows, which walks key blocks of 128; the CTA takes tiles in a
//           stride over a heaviest-first order
//   warp 0  TMA: Q per tile (double-buffered), K_j and V_j (double-buffered rings)
//   warp 1  tensor-memory allocation; lane 0 issues
//             S_j = Q K_j^T   (M=128, N=128, K=64)  into S[j % 2] (TMEM)
//             O  += P_j V_j   (M=128, N=64,  K=128) into O (TMEM)
//   warps 2-5  one query row per thread: read S_j from TMEM, online softmax in
//             log2 units, write P_j (bf16 pairs) to tensor memory as the A operand
//             of the next MMA, rescale O in TMEM when the row maximum grows by more
//             than 2^8 (otherwise the stale maximum is kept: p <= 256 is exact
//             enough in fp32 and bf16), finally O / l and the log-sum-exp.
//
// Operands: Q, K are K-major (head dimension contiguous); V is used as stored
// ([key][head dim]) as an MN-major B operand; P is read from tensor memory.
// Shared tiles use the 128-byte swizzle (rows of 64 bf16). No cluster multicast.
#pragma once
#include "common.cuh"

namespace attn_tc {

constexpr int BQ = 128, BKV = 128, HD = 64;   // HD: the backward's head size (the forward is templated)
constexpr int kThreads = 192;
constexpr int STAGES = 2;
// Forward geometry for head size D (64 or 32): Q, K, V tiles of 128 rows of D
// bf16 (rows of 128 or 64 bytes, in the tensor core's 128- or 64-byte swizzled
// layout, which the TMA's swizzle of the same width writes). No alignment
// slack: without static shared memory the dynamic block starts on a 1 KB
// boundary (checked at run time). At most 99,328 bytes and 256 TMEM columns a
// CTA: two CTAs share an SM.
template <int D>
struct FwdGeom {
  static_assert(D == 64 || D == 32, "head size");
  static constexpr int ROW = D * 2;                       // bytes per tile row
  static constexpr int Q_BYTES = BQ * ROW;
  static constexpr int KV_BYTES = BKV * ROW;
  static constexpr int SMEM_BYTES = 2 * Q_BYTES + STAGES * 2 * KV_BYTES + 1024 /*barriers*/;
  static constexpr uint64_t kSwizzle = D == 64 ? 2 : 4;  // descriptor layout: 128- / 64-byte swizzle
};
// Shared-memory matrix descriptor for a swizzled tile (layout 2: 128-byte rows,
// 4: 64-byte rows); strides in bytes.
GPT2_DEV uint64_t smem_desc_swz(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint64_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= layout << 61;
  return d;
}
constexpr int TMEM_COLS = 256;               // S [0,128), O [128,192), P [192,256); two CTAs share an SM
constexpr uint32_t S_COL0 = 0, O_COL = 128, P_COL = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;    // log2(256)


GPT2_DEV void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T (A: M rows in TMEM lanes, K along columns as bf16 pairs).
GPT2_DEV void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

GPT2_DEV void tmem_st32_u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
GPT2_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Load 16 consecutive fp32 columns of this warp's 32 TMEM lanes.
GPT2_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse,
                       int T, int H, int BH, float scale, int* err) {
  using G = FwdGeom<D>;
  constexpr int HD = D;
  constexpr int Q_BYTES = G::Q_BYTES, KV_BYTES = G::KV_BYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw_af[];
  uint8_t* smem = smem_raw_af;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1 KB-aligned base
    if (threadIdx.x == 0) atomicOr(err, DEVERR_TIMEOUT);
    return;
  }
  uint8_t* sQ = smem;                          // [2][Q_BYTES]
  uint8_t* sK = sQ + 2 * Q_BYTES;              // [STAGES][KV_BYTES]
  uint8_t* sV = sK + STAGES * KV_BYTES;        // [STAGES][KV_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + STAGES * KV_BYTES);
  uint64_t* q_full = bars;         // [2]  Q of a tile landed
  uint64_t* q_empty = bars + 2;    // [2]  the tile's last S computed: Q buffer free
  uint64_t* k_full = bars + 4;     // [2]  K_j landed
  uint64_t* k_empty = bars + 6;    // [2]  S_j computed: K stage free
  uint64_t* v_full = bars + 8;     // [2]
  uint64_t* v_empty = bars + 10;   // [2]  P_j V_j computed: V stage free
  uint64_t* s_full = bars + 12;
  uint64_t* s_empty = bars + 13;
  uint64_t* p_full = bars + 14;
  uint64_t* p_empty = bars + 15;
  uint64_t* o_done = bars + 16;
  uint64_t* done = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = T / BQ;
  const int n_tiles = nqb * BH;
  const int C = H * HD;
  // Persistent: tile t is query block nqb - 1 - t / BH (the heaviest first) of
  // (batch, head) t % BH. In pass r the CTAs take tiles r G .. r G + G - 1
  // (G CTAs), in reversed order in odd passes, so that a CTA that drew a heavy
  // tile draws a light one next (over 8 query blocks the busiest CTA gets ~29
  // key blocks against a mean of 27.7; a plain stride gives it 32). Key blocks
  // are counted across the CTA's tiles (gb), so the K/V rings and the S, P and
  // O barriers run on without a reset between tiles.
  // the CTA's tile after tile t (the one it takes in the next pass)
  auto next_tile = [](int t) {
    const int r = t / (int)gridDim.x + 1;
    return r * (int)gridDim.x + ((r & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&q_full[i]), 1);
      mbar_init(smem_u32(&q_empty[i]), 1);
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_empty), 128);
    mbar_init(smem_u32(p_full), 128);
    mbar_init(smem_u32(p_empty), 1);
    mbar_init(smem_u32(o_done), 1);
    mbar_init(smem_u32(done), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();   // set-up above overlaps the previous kernel's drain

  if (warp == 0) {
    // -------------------------------------------------------------- TMA producer
    if (lane == 0) {
      // K and V run as separate two-deep rings: K_j is released once S_j is
      // computed, V_j once P_j V_j is, so K runs further ahead than V. Q is
      // double-buffered: the next tile's Q loads while this tile still runs.
      int gk = 0;   // key blocks of earlier tiles (ring positions)
      bool ok = true;
      for (int t = blockIdx.x, it = 0; t < n_tiles && ok; t = next_tile(t)) {
        const int qb = nqb - 1 - t / BH, bh = t % BH;
        const int b = bh / H, h = bh % H;
        const int row_base = b * T, nkv = qb + 1;
        const int qs = it & 1;
        if (it >= 2 && !mbar_wait(smem_u32(&q_empty[qs]), ((it >> 1) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(smem_u32(&q_full[qs]), Q_BYTES);
        tma_load_2d(smem_u32(sQ + qs * Q_BYTES), &tm_qkv, smem_u32(&q_full[qs]), h * HD, row_base + qb * BQ);
        int nk = 0, nv = 0;
        unsigned long long t0 = globaltimer_ns();
        while (nk < nkv || nv < nkv) {
          bool progressed = false;
          const int uk = gk + nk;
          if (nk < nkv && (uk < 2 || mbar_try_wait(smem_u32(&k_empty[uk & 1]), ((uk >> 1) & 1) ^ 1))) {
            const int st = uk & 1;
            mbar_arrive_expect_tx(smem_u32(&k_full[st]), KV_BYTES);
            tma_load_2d(smem_u32(sK + st * KV_BYTES), &tm_qkv, smem_u32(&k_full[st]), C + h * HD,
                        row_base + nk * BKV);
            ++nk;
            progressed = true;
          }
          const int uv = gk + nv;
          if (nv < nkv && nv < nk && (uv < 2 || mbar_try_wait(smem_u32(&v_empty[uv & 1]), ((uv >> 1) & 1) ^ 1))) {
            const int st = uv & 1;
            mbar_arrive_expect_tx(smem_u32(&v_full[st]), KV_BYTES);
            tma_load_2d(smem_u32(sV + st * KV_BYTES), &tm_qkv, smem_u32(&v_full[st]), 2 * C + h * HD,
                        row_base + nv * BKV);
            ++nv;
            progressed = true;
          }
          if (progressed) {
            t0 = globaltimer_ns();
          } else {
            if (*(volatile int*)err & DEVERR_TIMEOUT) { ok = false; break; }
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
              atomicOr(err, DEVERR_TIMEOUT);
              ok = false;
              break;
            }
          }
        }
        gk += nkv;
        ++it;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BQ, BKV, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(BQ, HD, false, true);
      // S_g = Q K_g^T for key block g (K ring position g) with Q buffer qs
      auto issue_s = [&](int g, int qs) {
        const int st = g & 1;
        const uint32_t q_addr = smem_u32(sQ + qs * Q_BYTES);
        const uint32_t k_addr = smem_u32(sK + st * KV_BYTES);
        const uint32_t d = tmem + S_COL0;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)   // K-major Q, K: 16 head-dim columns (32 bytes) a step
          tc_mma_bf16(d, smem_desc_swz(q_addr + kk * 32, 16, 8 * G::ROW, G::kSwizzle),
                      smem_desc_swz(k_addr + kk * 32, 16, 8 * G::ROW, G::kSwizzle), idesc_s, kk > 0 ? 1u : 0u);
        tc_commit(smem_u32(s_full));
        tc_commit(smem_u32(&k_empty[st]));
      };
      bool ok = true;
      if (blockIdx.x < n_tiles) {   // the first pass gives every CTA a tile
        ok = mbar_wait(smem_u32(&q_full[0]), 0, err) && mbar_wait(smem_u32(&k_full[0]), 0, err);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
        }
      }
      int gb = 0;   // key blocks issued in earlier iterations
      for (int t = blockIdx.x, it = 0; t < n_tiles && ok; t = next_tile(t)) {
        const int nkv = nqb - t / BH;   // causal: key blocks 0..qb
        const bool more = next_tile(t) < n_tiles;
        for (int j = 0; j < nkv; ++j, ++gb) {
          // S of the next key block: this tile's next one, or the next tile's first,
          // once its K landed and the softmax has taken S_gb out of tensor memory
          const bool last = (j + 1 == nkv);
          if (last) tc_commit(smem_u32(&q_empty[it & 1]));   // this tile's last S read Q
          if (!last || more) {
            const int gn = gb + 1;
            int qs = it & 1;
            if (!mbar_wait(smem_u32(&k_full[gn & 1]), (gn >> 1) & 1, err)) { ok = false; break; }
            if (!mbar_wait(smem_u32(s_empty), gb & 1, err)) { ok = false; break; }
            if (last) {
              qs = (it + 1) & 1;
              if (!mbar_wait(smem_u32(&q_full[qs]), ((it + 1) >> 1) & 1, err)) { ok = false; break; }
            }
            tc_fence_after();
            issue_s(gn, qs);
          }
          // P_gb written (and O rescaled if needed)
          const int st = gb & 1;
          if (!mbar_wait(smem_u32(p_full), gb & 1, err)) { ok = false; break; }
          if (!mbar_wait(smem_u32(&v_full[st]), (gb >> 1) & 1, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sV + st * KV_BYTES);
          // V as stored ([key][head dim]): an MN-major B operand whose 8-key groups are
          // 8 rows apart; its head dimension is one swizzle atom wide
          const uint64_t vd = smem_desc_swz(v_addr, D == 64 ? 8192 : 8 * G::ROW, 8 * G::ROW, G::kSwizzle);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)   // A = P from tensor memory, 16 keys = 8 columns a step
            tc_mma_bf16_ts(tmem + O_COL, tmem + P_COL + kk * 8, vd + kk * ((16 * G::ROW) >> 4), idesc_o,
                           (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_u32(p_empty));
          tc_commit(smem_u32(&v_empty[st]));
          tc_commit(smem_u32(o_done));
        }
        ++it;
      }
      tc_commit(smem_u32(done));
      mbar_wait(smem_u32(done), 0, err);
    }
  } else {
    // -------------------------------------------------------------- softmax / epilogue
    const int q4 = warp & 3;                        // TMEM lane quarter
    const int r = q4 * 32 + lane;                   // query row within the tile
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = scale * kLog2e;
    bool ok = true;
    int gb = 0;   // key blocks of earlier tiles and of this one so far
    for (int t = blockIdx.x; t < n_tiles && ok; t = next_tile(t)) {
      const int qb = nqb - 1 - t / BH;
      const int nkv = qb + 1;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j, ++gb) {
        if (!mbar_wait(smem_u32(s_full), gb & 1, err)) { ok = false; break; }
        tc_fence_after();
        const bool diag = (j == qb);
        const uint32_t s_tm = tmem + lane_off + S_COL0;
        // the whole score row (128 fp32) in four loads, one wait; S is free again at once
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_async(s_tm + c * 32, sr[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(smem_u32(s_empty));
        if (diag) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > r) sr[c][i] = __float_as_uint(-INFINITY);
        }
        // row maximum with eight independent partial maxima (short dependency
        // chains), two scores per three-input max
        float mpart[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mpart[u] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mpart[(i >> 1) & 7] =
                max3f(mpart[(i >> 1) & 7], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
        const float mx = max3f(max3f(mpart[0], mpart[1], mpart[2]), max3f(mpart[3], mpart[4], mpart[5]),
                               fmaxf(mpart[6], mpart[7])) *
                         sl2;  // scale > 0: max commutes with it
        // lazy rescale: keep the stale maximum unless the new one exceeds it by > 2^8
        const bool grow = (mx > m + kRescaleThreshold) || (m == -INFINITY);
        const float m_new = grow ? mx : m;
        const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
        // four paired partial sums; the scale-and-shift and the sums run as paired
        // fp32 operations (two scores per instruction)
        float2 spart[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) spart[u] = make_float2(0.f, 0.f);
        const float2 sl2x2 = make_float2(sl2, sl2), negm2 = make_float2(-m_new, -m_new);
        // P as bf16 pairs (keys 2i, 2i+1 of this query row in column P_COL + i),
        // in two halves of 64 keys: the first half's 32 words are stored (once the
        // PV product of the previous key block has read the P buffer) before the
        // second half is formed, so only 32 packed words are live at a time
        bool waited = false;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 y = f2_fma(make_float2(__uint_as_float(sr[c][2 * i]), __uint_as_float(sr[c][2 * i + 1])),
                                      sl2x2, negm2);
              const float2 pp = make_float2(ex2_approx(y.x), ex2_approx(y.y));
              spart[i & 3] = f2_add(spart[i & 3], pp);
              pk[cc * 16 + i] = pack_bf16x2(pp.x, pp.y);
            }
          }
          if (!waited) {
            // the P buffer was last read by the PV product of key block gb - 1
            if (gb >= 1 && !mbar_wait(smem_u32(p_empty), (gb - 1) & 1, err)) { ok = false; }
            tc_fence_after();
            waited = true;
          }
          if (ok) tmem_st32_u(tmem + lane_off + P_COL + 32 * half, pk);
        }
        if (!ok) break;
        const float2 s01 = f2_add(spart[0], spart[1]), s23 = f2_add(spart[2], spart[3]);
        const float2 s4 = f2_add(s01, s23);
        const float sum = s4.x + s4.y;
        l = l * alpha + sum;
        m = m_new;
        // O rescale (rows whose maximum moved) once the PV product of key block gb - 1 is done
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          if (!mbar_wait(smem_u32(o_done), (gb - 1) & 1, err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            float v[32];
            tmem_ld32(tmem + lane_off + O_COL + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st32(tmem + lane_off + O_COL + c * 32, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(p_full));
      }
      if (!ok) break;
      // epilogue: O / l, log-sum-exp, once the tile's last PV product is done; O is
      // read out before this warp's next P is posted, so the next tile's first PV
      // product (which overwrites O) cannot start earlier
      if (!mbar_wait(smem_u32(o_done), (gb - 1) & 1, err)) break;
      tc_fence_after();
      const int bh = t % BH;
      const int qrow = qb * BQ + r;                 // query position
      const float inv = 1.0f / l;
      bf16* orow = out + ((size_t)((bh / H) * T + qrow)) * C + (bh % H) * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_off + O_COL + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          *reinterpret_cast<uint4*>(orow + c * 32 + i) =
              make_uint4(pack_bf16x2(v[i] * inv, v[i + 1] * inv), pack_bf16x2(v[i + 2] * inv, v[i + 3] * inv),
                         pack_bf16x2(v[i + 4] * inv, v[i + 5] * inv), pack_bf16x2(v[i + 6] * inv, v[i + 7] * inv));
      }
      lse[(size_t)bh * T + qrow] = (m + log2f(l)) * kLn2;
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// qkv bf16 [B*T, 3C] (q | k | v, heads contiguous), out bf16 [B*T, C], lse fp32 [B, H, T];
// head size D = 64 or 32, T a multiple of 128.
template <int D>
static cudaError_t fwd(const bf16* qkv, bf16* out, float* lse, int B, int T, int H, int* err, cudaStream_t s) {
  using G = FwdGeom<D>;
  static PerDeviceOnce once;
  cudaError_t e0 = once.run([] {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // ask for the whole shared-memory carveout so that two CTAs share an SM
    return cudaFuncSetAttribute(attn_fwd_tc_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (e0 != cudaSuccess) return e0;
  if (T % BQ) return cudaErrorInvalidValue;
  const int C = H * D;
  CUtensorMap tm;
  if (!encode_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, 3 * (uint64_t)C, (uint64_t)B * T, 3 * (uint64_t)C,
                     D, 128, D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  // persistent: two CTAs an SM, or one per tile if there are fewer tiles
  const int n_tiles = (T / BQ) * B * H;
  const int grid = std::min(n_tiles, 2 * device_sm_count());
  launch_pdl(attn_fwd_tc_kernel<D>, dim3(grid), dim3(kThreads), G::SMEM_BYTES, s, tm, out, lse, T, H, B * H,
             1.0f / sqrtf((float)D), err);
  return cudaGetLastError();
}


// ===========================================================================
// Backward (head size 64). Three kernels:
//
//   bwd_prep_kernel   per (batch, head, query): D = rowsum(dO o O) (the softmax
//                     Jacobian term); writes -lse/scale and -D, each as a bf16
//                     hi + lo pair, into a 16-column operand tile per query block
//                     (see below); clears the fp32 dQ accumulator.
//   attn_bwd_tc_kernel  persistent, one CTA per SM; a work item is one (batch,
//                     head) and a block of 128 keys, which walks the query blocks
//                     at or after it (causal). The next item's K, V load as soon as
//                     the last product of the current one has read them, so one
//                     item's epilogue overlaps the next one's first loads. With
//                     K, V resident and Q_i, dO_i streamed through a three-deep ring:
//       S'^T  = [K | 1 1 0..] [Q_i | X_i]^T   = S^T - lse/scale  (M=128 keys, N=128 queries,
//       dP'^T = [V | 0 0 1 1 0..] [dO_i | X_i]^T = dP^T - D       K = 64 + one 16-wide step)
//       P^T  = exp2(S'^T * scale*log2e)       (softmax warps, one key row each)
//       dS^T = P^T * dP'^T * scale
//     where X_i holds (hi, lo) of -lse/scale and of -D per query: the per-query
//     terms enter through the tensor core, so the softmax warps read no shared
//     memory (their loads would queue behind the tensor core's operand reads).
//       dV  += P^T dO_i   (A = P^T from tensor memory)   (M=128 keys, N=64, K=128)
//       dK  += dS^T Q_i   (A = dS^T from shared memory)
//       dQ_i = dS K       (A = dS^T read MN-major)       (M=128 queries, N=64, K=128)
//     S^T/dP^T of query block i+1 are issued before the dV/dK/dQ products of
//     block i, so the tensor cores work on block i while the softmax warps turn
//     block i+1's scores into P and dS. Each softmax warp moves its 32 x 32
//     quarter of dQ_i out of tensor memory and adds it into the fp32
//     accumulator with its own TMA bulk reduce (no block-wide barrier).
//   bwd_post_kernel   dQ accumulator (fp32) -> the q third of dqkv (bf16).
//
// The softmax scale 1/8 is a power of two, so folding it into dS (bf16) is
// exact: dK and dQ need no rescale.
// TMEM: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384), dQ [384,448),
//       P^T as bf16 pairs [448,512).
// ===========================================================================
namespace bwd {
constexpr int BKEY = 128, BQRY = 128;
constexpr int NQS = 3;                              // Q / dO ring depth
constexpr int DST_BYTES = BKEY * BQRY * 2;          // 32 KB: dS^T
constexpr int DQW_BYTES = 32 * 32 * 4;              // 4 KB: one warp's dQ staging box
constexpr int kSoftmaxWarps = 8;
// warpgroup 0: TMA (warp 0), MMA (warp 1), two idle warps; warpgroups 1-2: softmax.
// Launched at 168 registers a thread (three warps per scheduler), warpgroup 0
// gives registers to the softmax warpgroups: 128 x 40 + 256 x 232 = 384 x 168.
constexpr int kThreads = 128 + 32 * kSoftmaxWarps;
constexpr int kLaunchRegs = 168, kCtlRegs = 152, kSoftmaxRegs = 176;
static_assert(128 * kCtlRegs + 32 * kSoftmaxWarps * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr int XT_BYTES = 128 * 16 * 2;              // 4 KB: a 128 x 16 extra-K operand tile
// The constant extra-K tiles of K' and V' have 128 identical rows: one 8-row
// group (two core matrices, 256 bytes) serves every row group through a
// descriptor whose row-group stride is 0.
constexpr int XC_BYTES = 256;
// Per head size D (64 or 32): a 128-row tile of K, V, Q or dO has rows of 2 D
// bytes in the 128- or 64-byte swizzled layout.
template <int D>
struct Geom {
  static constexpr int ROW = D * 2;
  static constexpr int T_BYTES = 128 * ROW;
  // K has two buffers (the next item's K loads while this item runs), V one
  // (it is released once an item's last scores are computed). No alignment
  // slack: without static shared memory the dynamic block starts on a 1 KB
  // boundary (checked at run time).
  static constexpr int SMEM_BYTES = 3 * T_BYTES /*K x2, V*/ + NQS * 2 * T_BYTES /*Q,dO*/ + DST_BYTES +
                                    kSoftmaxWarps * DQW_BYTES + NQS * XT_BYTES /*X_i*/ +
                                    2 * XC_BYTES /*K', V' columns*/ + 256 /*barriers*/;
  static constexpr uint64_t kSwizzle = D == 64 ? 2 : 4;
  static constexpr uint32_t kMnLbo = D == 64 ? 8192 : 8 * ROW;   // MN-major: one swizzle atom wide, unused
};
constexpr uint32_t C_S = 0, C_DP = 128, C_DV = 256, C_DK = 320, C_DQ = 384, C_P = 448;
constexpr int TMEM_COLS_BWD = 512;
constexpr int kPrepRows = 64;                       // query rows per prep block
constexpr int kMaxHeads = 64;
}  // namespace bwd

// Extra-K operand tiles (128 rows x 16 bf16) use the tensor core's non-swizzled
// K-major layout: 8-row x 16-byte core matrices stored as 128 contiguous bytes,
// the two core matrices of a row group adjacent (128 bytes apart along K) and
// row groups 256 bytes apart. Byte offset of (row, col):
__host__ __device__ constexpr int xt_offset(int row, int col) {
  return ((row >> 3) * 2 + (col >> 3)) * 128 + (row & 7) * 16 + (col & 7) * 2;
}
GPT2_DEV uint64_t smem_desc_interleave(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100; layout 0: no swizzle
  return d;
}

GPT2_DEV void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}


template <int N>
GPT2_DEV void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
GPT2_DEV void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// P^T and dS^T of one key row (this thread) for 64 query columns. DIAG: the
// query block is the key block itself, so keys after the query are masked.
template <bool DIAG>
GPT2_DEV void bwd_softmax_row(const uint32_t (&sv)[2][32], const uint32_t (&dv)[2][32], float sl2, float scale,
                              int r, int col0, uint32_t (&pp)[32], uint32_t (&pd)[32]) {
  // two columns per paired fp32 instruction
  const float2 sl2x2 = make_float2(sl2, sl2), sc2 = make_float2(scale, scale);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      const int j = 2 * g;   // column pair within this 32-column chunk
      // S' already holds -lse/scale, dP' already holds -D
      const float2 y = f2_mul(make_float2(__uint_as_float(sv[c][j]), __uint_as_float(sv[c][j + 1])), sl2x2);
      float2 p = make_float2(ex2_approx(y.x), ex2_approx(y.y));
      if (DIAG) {   // key after query: masked
        if (r > col0 + c * 32 + j) p.x = 0.f;
        if (r > col0 + c * 32 + j + 1) p.y = 0.f;
      }
      const float2 ds =
          f2_mul(p, f2_mul(make_float2(__uint_as_float(dv[c][j]), __uint_as_float(dv[c][j + 1])), sc2));
      pp[c * 16 + g] = pack_bf16x2(p.x, p.y);
      pd[c * 16 + g] = pack_bf16x2(ds.x, ds.y);
    }
  }
}

// Block: 64 consecutive query rows of one sequence, all heads, in
// 32 * ceil(C/256) * RW threads, RW = max(1, 12 / ceil(C/256)). Warp w takes
// the 32 16-byte chunks of group g = w % ceil(C/256) (lanes hold chunks of O
// and dO, D / 8 chunks per head) in the rows rl = w / ceil(C/256) + RW i.
// With dbias_v the block also adds the column sums of its 64 rows of dO into
// dbias_v (fp32 [C], 16-byte aligned): the gradient of the value bias, since
// every row of causal softmax weights sums to one (an output row is a convex
// combination of value rows, so a bias added to every value row passes through
// unchanged). A lane keeps its chunk's sums over its rows in registers; the RW
// row warps of a chunk group are added once through shared memory.
template <int D>
__global__ void __launch_bounds__(512) bwd_prep_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                                       const float* __restrict__ lse, uint8_t* __restrict__ xtiles,
                                                       float* __restrict__ dq_acc, float* __restrict__ dbias_v, int T,
                                                       int H, float scale) {
  pdl_begin();
  using namespace bwd;
  constexpr int CPH = D / 8;                 // 16-byte chunks per head
  __shared__ float sDot[kMaxHeads][kPrepRows];
  __shared__ __align__(16) float sPart[512 * 8];
  const int C = H * D;
  const int NV = C / 8;                      // 16-byte chunks per row
  const int NG = (NV + 31) / 32;             // chunk groups of 32
  const int RW = (blockDim.x >> 5) / NG;     // row warps per chunk group (the host makes this >= 1)
  const int row0 = blockIdx.x * kPrepRows;   // global row (b*T + t) of the first query
  const int b = row0 / T, t0 = row0 % T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = warp % NG, rw = warp / NG;
  const int vi = g * 32 + lane;
  float cs[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) cs[k] = 0.f;
  if (rw < RW) {
#pragma unroll 4
    for (int rl = rw; rl < kPrepRows; rl += RW) {
      const size_t base = (size_t)(row0 + rl) * C;
      float acc = 0.f;
      if (vi < NV) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(out + base) + vi);
        const uint4 c = __ldg(reinterpret_cast<const uint4*>(dout + base) + vi);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 fa = unpack_bf16x2(aw[k]), fc = unpack_bf16x2(cw[k]);
          acc = fmaf(fa.x, fc.x, fmaf(fa.y, fc.y, acc));
          cs[2 * k] += fc.x;
          cs[2 * k + 1] += fc.y;
        }
      }
#pragma unroll
      for (int o = 1; o < CPH; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if ((lane & (CPH - 1)) == 0 && vi < NV) sDot[vi / CPH][rl] = acc;
    }
  }
  const bool colsum = dbias_v != nullptr;
  if (colsum && rw < RW && vi < NV) {
    float4* sp = reinterpret_cast<float4*>(sPart + (rw * NG * 32 + vi) * 8);
    sp[0] = make_float4(cs[0], cs[1], cs[2], cs[3]);
    sp[1] = make_float4(cs[4], cs[5], cs[6], cs[7]);
  }
  __syncthreads();
  if (colsum)
    for (int i = threadIdx.x; i < C / 4; i += blockDim.x) {   // i: a group of four columns
      float4 s4 = reinterpret_cast<const float4*>(sPart)[i];
      for (int r = 1; r < RW; ++r) {
        const float4 u = reinterpret_cast<const float4*>(sPart)[r * NG * 64 + i];
        s4.x += u.x; s4.y += u.y; s4.z += u.z; s4.w += u.w;
      }
      red_add_f32x4(dbias_v + 4 * i, s4.x, s4.y, s4.z, s4.w);
    }
  // X tile of query block (b, h, t / 128), row t % 128: columns 0,1 = (hi, lo) of
  // -lse/scale, columns 2,3 = (hi, lo) of -D, the rest 0
  for (int i = threadIdx.x; i < H * kPrepRows; i += blockDim.x) {
    const int h = i / kPrepRows, rl = i % kPrepRows;
    const int t = t0 + rl;
    const size_t o = ((size_t)b * H + h) * T + t;
    const float x1 = -lse[o] / scale, x2 = -sDot[h][rl];
    const float h1 = __bfloat162float(__float2bfloat16_rn(x1)), h2 = __bfloat162float(__float2bfloat16_rn(x2));
    uint8_t* tile = xtiles + (((size_t)b * H + h) * (T / BQRY) + t / BQRY) * XT_BYTES;
    const int qr = t % BQRY;
    *reinterpret_cast<uint4*>(tile + xt_offset(qr, 0)) =
        make_uint4(pack_bf16x2(h1, x1 - h1), pack_bf16x2(h2, x2 - h2), 0u, 0u);
    *reinterpret_cast<uint4*>(tile + xt_offset(qr, 8)) = make_uint4(0u, 0u, 0u, 0u);
  }
  float4* z = reinterpret_cast<float4*>(dq_acc + (size_t)row0 * C);
  const int n4 = kPrepRows * C / 4;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dq_acc fp32 [rows, C] -> dqkv[:, 0:C] bf16 (row stride 3C), in blocks of
// (C/8) * RL threads: thread t of block b converts the eight columns of chunk
// t % (C/8) in rows (b RL + t / (C/8)) + k gridDim.x RL, so that the grid
// sweeps the matrix as one contiguous band. With dbias_q the block adds the
// column sums of its rows of dQ (fp32, before rounding) into dbias_q (fp32
// [C], 16-byte aligned): the query bias gradient.
__global__ void __launch_bounds__(1024) bwd_post_kernel(const float* __restrict__ dq_acc, bf16* __restrict__ dqkv,
                                                        float* __restrict__ dbias_q, int rows, int C) {
  pdl_begin();
  __shared__ __align__(16) float sPart[1024 * 8];
  const int NV = C / 8;
  const int RL = blockDim.x / NV;             // row lanes (the host makes this >= 1)
  const int c8 = threadIdx.x % NV, rl = threadIdx.x / NV;
  const int band = gridDim.x * RL;
  float cs[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) cs[k] = 0.f;
  if (rl < RL) {
#pragma unroll 4
    for (int row = blockIdx.x * RL + rl; row < rows; row += band) {
      const float4* src = reinterpret_cast<const float4*>(dq_acc + (size_t)row * C + c8 * 8);
      const float4 a = __ldcs(src), c = __ldcs(src + 1);
      *reinterpret_cast<uint4*>(dqkv + (size_t)row * 3 * C + c8 * 8) =
          make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
      cs[0] += a.x; cs[1] += a.y; cs[2] += a.z; cs[3] += a.w;
      cs[4] += c.x; cs[5] += c.y; cs[6] += c.z; cs[7] += c.w;
    }
  }
  if (dbias_q == nullptr) return;
  // the RL row lanes' sums of each chunk, added in a fixed order, then one
  // vector atomic per four columns
  float4* sp = reinterpret_cast<float4*>(sPart);
  if (rl < RL) {
    sp[2 * threadIdx.x] = make_float4(cs[0], cs[1], cs[2], cs[3]);
    sp[2 * threadIdx.x + 1] = make_float4(cs[4], cs[5], cs[6], cs[7]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * NV; i += blockDim.x) {   // i: a group of four columns
    float4 s4 = sp[i];
    for (int r = 1; r < RL; ++r) {
      const float4 u = sp[r * 2 * NV + i];
      s4.x += u.x; s4.y += u.y; s4.z += u.z; s4.w += u.w;
    }
    red_add_f32x4(dbias_q + 4 * i, s4.x, s4.y, s4.z, s4.w);
  }
}

template <int D>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dq, const uint8_t* __restrict__ xtiles,
                       bf16* __restrict__ dqkv, int T, int H, int BH, float scale, int* err) {
  using namespace bwd;
  using G = Geom<D>;
  constexpr int HD = D;
  constexpr int T_BYTES = G::T_BYTES;
  constexpr int NO = D / 2;                       // head-dim columns of dQ, dK, dV per softmax warp
  extern __shared__ __align__(1024) uint8_t smem_raw_ab[];
  uint8_t* smem = smem_raw_ab;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1 KB-aligned base
    if (threadIdx.x == 0) atomicOr(err, DEVERR_TIMEOUT);
    return;
  }
  uint8_t* sK = smem;                             // [2]
  uint8_t* sV = sK + 2 * T_BYTES;
  uint8_t* sQ = sV + T_BYTES;                     // [NQS]
  uint8_t* sDO = sQ + NQS * T_BYTES;              // [NQS]
  uint8_t* sDST = sDO + NQS * T_BYTES;
  uint8_t* sDQW = sDST + DST_BYTES;               // [kSoftmaxWarps][DQW_BYTES]
  uint8_t* sXQ = sDQW + kSoftmaxWarps * DQW_BYTES;  // [NQS] X_i tiles
  uint8_t* sXK = sXQ + NQS * XT_BYTES;              // K' extra columns: 1 1 0 ..
  uint8_t* sXV = sXK + XC_BYTES;                    // V' extra columns: 0 0 1 1 0 ..
  uint64_t* bars = reinterpret_cast<uint64_t*>(sXV + XC_BYTES);
  uint64_t* k_full = bars;                // [2]
  uint64_t* k_empty = bars + 2;           // [2]
  uint64_t* v_full = bars + 4;
  uint64_t* v_empty = bars + 5;
  uint64_t* qdo_full = bars + 6;          // [NQS]
  uint64_t* qdo_empty = bars + 6 + NQS;   // [NQS]
  uint64_t* st_full = bars + 6 + 2 * NQS;
  uint64_t* st_empty = st_full + 1;
  uint64_t* ds_full = st_full + 2;
  uint64_t* ds_empty = st_full + 3;
  uint64_t* dq_full = st_full + 4;
  uint64_t* dq_empty = st_full + 5;
  uint64_t* dkdv_full = st_full + 6;
  uint64_t* dkdv_empty = st_full + 7;
  uint64_t* done = st_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(st_full + 9);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = T / BKEY;
  const int C = H * HD;
  // Persistent: item i is key block i / BH of (batch, head) i % BH, so the
  // heaviest key blocks (kb = 0: every query block) come first; in pass r the
  // CTAs take items r G .. r G + G - 1 (G CTAs), in reversed order in odd
  // passes, so that a CTA that drew a heavy item draws a light one next (the
  // busiest CTA gets ~56 query blocks against a mean of 55.5 at 8 key blocks,
  // 148 CTAs; a plain stride gives it 60). Barrier phases run over g, the CTA's
  // count of query blocks processed, and over j, its count of items.
  const int n_items = nb * BH;
  auto next_item = [](int i) {   // the CTA's item after item i
    const int r = i / (int)gridDim.x + 1;
    return r * (int)gridDim.x + ((r & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
    }
    mbar_init(smem_u32(v_full), 1);
    mbar_init(smem_u32(v_empty), 1);
    for (int i = 0; i < NQS; ++i) {
      mbar_init(smem_u32(&qdo_full[i]), 1);
      mbar_init(smem_u32(&qdo_empty[i]), 1);
    }
    mbar_init(smem_u32(st_full), 1);
    mbar_init(smem_u32(st_empty), kSoftmaxWarps);
    mbar_init(smem_u32(ds_full), kSoftmaxWarps);
    mbar_init(smem_u32(ds_empty), 1);
    mbar_init(smem_u32(dq_full), 1);
    mbar_init(smem_u32(dq_empty), kSoftmaxWarps);
    mbar_init(smem_u32(dkdv_full), 1);
    mbar_init(smem_u32(dkdv_empty), kSoftmaxWarps);
    mbar_init(smem_u32(done), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  // constant extra-K columns of K' and V' (1.0 in bf16 is 0x3F80): one row group
  for (int i = threadIdx.x; i < 8 * 2; i += blockDim.x) {
    const int row = i >> 1, half = i & 1;
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4*>(sXK + xt_offset(row, 8 * half)) = make_uint4(half ? 0u : one2, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(sXV + xt_offset(row, 8 * half)) = make_uint4(0u, half ? 0u : one2, 0u, 0u);
  }
  fence_async_smem();
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS_BWD);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();   // set-up above overlaps the previous kernel's drain

  if (warp < 4) {
    regs_dec<kCtlRegs>();
    if (warp == 0) {
      // -------------------------------------------------------------- TMA producer
      if (lane == 0) {
        bool ok = true;
        int g = 0;
        auto load_qdo = [&](int gq, int bh, int row_base, int h, int qi) -> bool {
          const int s = gq % NQS, u = gq / NQS;
          if (!mbar_wait(smem_u32(&qdo_empty[s]), (u & 1) ^ 1, err)) return false;
          const uint32_t fb = smem_u32(&qdo_full[s]);
          mbar_arrive_expect_tx(fb, 2 * T_BYTES + XT_BYTES);
          tma_load_2d(smem_u32(sQ + s * T_BYTES), &tm_qkv, fb, h * HD, row_base + qi * BQRY);
          tma_load_2d(smem_u32(sDO + s * T_BYTES), &tm_do, fb, h * HD, row_base + qi * BQRY);
          bulk_load_1d(smem_u32(sXQ + s * XT_BYTES), xtiles + ((size_t)bh * nb + qi) * XT_BYTES, XT_BYTES, fb);
          return true;
        };
        for (int i = blockIdx.x, j = 0; i < n_items && ok; i = next_item(i), ++j) {
          const int kb = i / BH, bh = i % BH, b = bh / H, h = bh % H;
          const int row_base = b * T, nit = nb - kb;
          // the first query block of this item may land before its keys
          ok = load_qdo(g, bh, row_base, h, kb);
          // V once the previous item's last scores have been computed
          if (ok && j > 0 && !mbar_wait(smem_u32(v_empty), (j - 1) & 1, err)) ok = false;
          if (!ok) break;
          mbar_arrive_expect_tx(smem_u32(v_full), T_BYTES);
          tma_load_2d(smem_u32(sV), &tm_qkv, smem_u32(v_full), 2 * C + h * HD, row_base + kb * BKEY);
          if (j == 0) {   // later items' K is loaded one item ahead (below)
            mbar_arrive_expect_tx(smem_u32(&k_full[0]), T_BYTES);
            tma_load_2d(smem_u32(sK), &tm_qkv, smem_u32(&k_full[0]), C + h * HD, row_base + kb * BKEY);
          }
          for (int it = 1; it < nit && ok; ++it) ok = load_qdo(g + it, bh, row_base, h, kb + it);
          g += nit;
          // the next item's K into the other buffer, once the item before this
          // one has released it
          const int i2 = next_item(i);
          if (ok && i2 < n_items) {
            const int kb2 = i2 / BH, bh2 = i2 % BH, b2 = bh2 / H, h2 = bh2 % H;
            const int nbuf = (j + 1) & 1;
            if (j >= 1 && !mbar_wait(smem_u32(&k_empty[nbuf]), ((j - 1) >> 1) & 1, err)) { ok = false; break; }
            mbar_arrive_expect_tx(smem_u32(&k_full[nbuf]), T_BYTES);
            tma_load_2d(smem_u32(sK + nbuf * T_BYTES), &tm_qkv, smem_u32(&k_full[nbuf]), C + h2 * HD,
                        b2 * T + kb2 * BKEY);
          }
        }
      }
    } else if (warp == 1) {
      // -------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t id_st = idesc_bf16_f32(BKEY, BQRY, false, false);  // S^T, dP^T
        constexpr uint32_t id_kv = idesc_bf16_f32(BKEY, HD, false, true);     // dV (A in TMEM), dK
        constexpr uint32_t id_q = idesc_bf16_f32(BQRY, HD, true, true);       // dQ
        // Descriptors are formed once; a shared-memory offset is added in 16-byte
        // units to the start-address field (addresses stay below 2^18, no carry).
        constexpr uint32_t kSbo = 8 * G::ROW;                                 // 8-row groups
        const uint64_t dK_k = smem_desc_swz(smem_u32(sK), 16, kSbo, G::kSwizzle);        // K, K-major
        const uint64_t dV_k = smem_desc_swz(smem_u32(sV), 16, kSbo, G::kSwizzle);        // V, K-major
        const uint64_t dK_mn = smem_desc_swz(smem_u32(sK), G::kMnLbo, kSbo, G::kSwizzle);  // K, MN-major
        const uint64_t dDS_k = smem_desc_sw128(smem_u32(sDST), 16, 1024);     // dS^T, K-major
        const uint64_t dDS_mn = smem_desc_sw128(smem_u32(sDST), BKEY * 128, 1024);  // dS, MN-major
        const uint64_t dQ0_k = smem_desc_swz(smem_u32(sQ), 16, kSbo, G::kSwizzle);
        const uint64_t dQ0_mn = smem_desc_swz(smem_u32(sQ), G::kMnLbo, kSbo, G::kSwizzle);
        const uint64_t dO0_k = smem_desc_swz(smem_u32(sDO), 16, kSbo, G::kSwizzle);
        const uint64_t dO0_mn = smem_desc_swz(smem_u32(sDO), G::kMnLbo, kSbo, G::kSwizzle);
        constexpr uint64_t kMnStep = (16 * G::ROW) >> 4;   // 16 rows of an MN-major operand, descriptor units
        const uint64_t dXK = smem_desc_interleave(smem_u32(sXK), 128, 0);   // one row group for all
        const uint64_t dXV = smem_desc_interleave(smem_u32(sXV), 128, 0);
        constexpr uint64_t kKBuf = T_BYTES >> 4;   // the second K buffer, in descriptor units
        const uint64_t dXQ0 = smem_desc_interleave(smem_u32(sXQ), 128, 256);
        constexpr uint64_t kXStage = XT_BYTES >> 4;
        constexpr uint64_t kStage = T_BYTES >> 4;   // one Q/dO stage, in descriptor units
        auto issue_st = [&](int gq, uint64_t ko) {
          const uint64_t so = (uint64_t)(gq % NQS) * kStage;
          const uint64_t sx = (uint64_t)(gq % NQS) * kXStage;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            tc_mma_bf16(tmem + C_S, dK_k + ko + kk * 2, dQ0_k + so + kk * 2, id_st, kk > 0 ? 1u : 0u);
            tc_mma_bf16(tmem + C_DP, dV_k + kk * 2, dO0_k + so + kk * 2, id_st, kk > 0 ? 1u : 0u);
          }
          // the per-query terms: S^T - lse/scale, dP^T - D
          tc_mma_bf16(tmem + C_S, dXK, dXQ0 + sx, id_st, 1u);
          tc_mma_bf16(tmem + C_DP, dXV, dXQ0 + sx, id_st, 1u);
          tc_commit(smem_u32(st_full));
        };
        bool ok = true;
        int g = 0;
        for (int i = blockIdx.x, j = 0; i < n_items && ok; i = next_item(i), ++j) {
          const int nit = nb - i / BH;
          const uint64_t ko = (j & 1) ? kKBuf : 0;
          // this item's keys, its first query block, and the previous scores out of TMEM
          if (!mbar_wait(smem_u32(&k_full[j & 1]), (j >> 1) & 1, err)) { ok = false; break; }
          if (!mbar_wait(smem_u32(v_full), j & 1, err)) { ok = false; break; }
          if (!mbar_wait(smem_u32(&qdo_full[g % NQS]), (g / NQS) & 1, err)) { ok = false; break; }
          if (g > 0 && !mbar_wait(smem_u32(st_empty), (g - 1) & 1, err)) { ok = false; break; }
          tc_fence_after();
          issue_st(g, ko);
          if (nit == 1) tc_commit(smem_u32(v_empty));   // the item's last scores read V
          for (int it = 0; it < nit && ok; ++it) {
            const int gc = g + it;
            const uint64_t so = (uint64_t)(gc % NQS) * kStage;
            if (it + 1 < nit) {
              // block it+1's scores, once its Q/dO landed and block it's scores left TMEM
              if (!mbar_wait(smem_u32(&qdo_full[(gc + 1) % NQS]), ((gc + 1) / NQS) & 1, err)) { ok = false; break; }
              if (!mbar_wait(smem_u32(st_empty), gc & 1, err)) { ok = false; break; }
              tc_fence_after();
              issue_st(gc + 1, ko);
              if (it + 2 == nit) tc_commit(smem_u32(v_empty));   // the item's last scores read V
            }
            // P^T (tensor memory) and dS^T (shared memory) of block it are written
            if (!mbar_wait(smem_u32(ds_full), gc & 1, err)) { ok = false; break; }
            // the previous item's dK, dV have left tensor memory
            if (it == 0 && j > 0 && !mbar_wait(smem_u32(dkdv_empty), (j - 1) & 1, err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t acc0 = it > 0 ? 1u : 0u;
#pragma unroll
            for (int kk = 0; kk < BQRY / 16; ++kk) {
              const uint32_t aoff = ((kk >> 2) * (BKEY * 128) + (kk & 3) * 32) >> 4;
              tc_mma_bf16_ts(tmem + C_DV, tmem + C_P + kk * 8, dO0_mn + so + kk * kMnStep, id_kv,
                             kk > 0 ? 1u : acc0);
              tc_mma_bf16(tmem + C_DK, dDS_k + aoff, dQ0_mn + so + kk * kMnStep, id_kv, kk > 0 ? 1u : acc0);
            }
            // dQ of this block once the previous block's dQ has left tensor memory
            if (gc > 0 && !mbar_wait(smem_u32(dq_empty), (gc - 1) & 1, err)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < BKEY / 16; ++kk)
              tc_mma_bf16(tmem + C_DQ, dDS_mn + kk * 128, dK_mn + ko + kk * kMnStep, id_q, kk > 0 ? 1u : 0u);
            tc_commit(smem_u32(dq_full));
            tc_commit(smem_u32(ds_empty));
            tc_commit(smem_u32(&qdo_empty[gc % NQS]));
          }
          tc_commit(smem_u32(dkdv_full));   // this item's dK, dV are complete
          tc_commit(smem_u32(&k_empty[j & 1]));   // and its K buffer is no longer read
          g += nit;
        }
        // every product has completed before the block releases tensor memory
        tc_commit(smem_u32(done));
        mbar_wait(smem_u32(done), 0, err);
      }
    }
  } else {
    regs_inc<kSoftmaxRegs>();
    // -------------------------------------------------------------- softmax-backward warps
    // warps 4..11: TMEM lane quarter q4 = warp & 3 (key rows), query-column half hf
    const int q4 = warp & 3, hf = (warp - 4) >> 2, wi = warp - 4;
    const int r = q4 * 32 + lane;                  // key row (and query row for dQ)
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = scale * kLog2e;
    uint8_t* stage = sDQW + wi * DQW_BYTES;
    // dQ of query block gq (rows qrow0.., columns hc..): this warp's 32 query rows
    // x 32 columns -> staging box -> bulk reduce-add into the accumulator
    auto drain_dq = [&](int gq, int hc, int qrow0) -> bool {
      if (!mbar_wait(smem_u32(dq_full), gq & 1, err)) return false;
      tc_fence_after();
      float v[NO];
      if (NO == 32) tmem_ld32(tmem + lane_off + C_DQ + hf * NO, *reinterpret_cast<float(*)[32]>(v));
      else tmem_ld16(tmem + lane_off + C_DQ + hf * NO, *reinterpret_cast<float(*)[16]>(v));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(dq_empty));
        bulk_wait_group_read<0>();   // this warp's previous reduce has read the box
      }
      __syncwarp();
      // the staging box: 32 rows of NO floats in the reduce map's swizzled layout
      // (128-byte rows: chunk ^ (row & 7); 64-byte rows: chunk ^ ((row >> 1) & 3))
#pragma unroll
      for (int ch = 0; ch < NO / 4; ++ch) {
        const int pc = NO == 32 ? (ch ^ (lane & 7)) : (ch ^ ((lane >> 1) & 3));
        *reinterpret_cast<float4*>(stage + lane * (NO * 4) + (pc << 4)) =
            make_float4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_2d(&tm_dq, smem_u32(stage), hc + hf * NO, qrow0 + q4 * 32);
        bulk_commit_group();
      }
      return true;
    };
    bool ok = true;
    int g = 0;
    int prev_hc = 0, prev_qrow0 = 0;   // where the previous block's dQ goes
    for (int i = blockIdx.x, j = 0; i < n_items && ok; i = next_item(i), ++j) {
      const int kb = i / BH, bh = i % BH, b = bh / H, h = bh % H;
      const int row_base = b * T, nit = nb - kb;
      for (int it = 0; it < nit && ok; ++it) {
        const int gc = g + it;
        if (!mbar_wait(smem_u32(st_full), gc & 1, err)) { ok = false; break; }
        tc_fence_after();
        // this thread's 64 query columns of S'^T and dP'^T; tensor memory is free again at once
        uint32_t sv[2][32], dv[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32_async(tmem + lane_off + C_S + hf * 64 + c * 32, sv[c]);
          tmem_ld32_async(tmem + lane_off + C_DP + hf * 64 + c * 32, dv[c]);
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(st_empty));
        uint32_t pp[32], pd[32];
        if (it == 0) bwd_softmax_row<true>(sv, dv, sl2, scale, r, hf * 64, pp, pd);
        else bwd_softmax_row<false>(sv, dv, sl2, scale, r, hf * 64, pp, pd);
        // P^T (TMEM) and dS^T (smem) were last read by the products of the previous block
        if (gc > 0 && !mbar_wait(smem_u32(ds_empty), (gc - 1) & 1, err)) { ok = false; break; }
        tc_fence_after();
        tmem_st32_u(tmem + lane_off + C_P + hf * 32, pp);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int off = hf * (BKEY * 128) + r * 128 + ((ch ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(sDST + off) = make_uint4(pd[4 * ch], pd[4 * ch + 1], pd[4 * ch + 2], pd[4 * ch + 3]);
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(ds_full));
        // while the products of this block run, move the previous block's dQ out
        if (gc > 0 && !drain_dq(gc - 1, prev_hc, prev_qrow0)) { ok = false; break; }
        prev_hc = h * HD;
        prev_qrow0 = row_base + (kb + it) * BQRY;
      }
      if (!ok) break;
      g += nit;
      // dK, dV of this item for key row r, head-dim columns 32 hf ..
      if (!mbar_wait(smem_u32(dkdv_full), j & 1, err)) { ok = false; break; }
      tc_fence_after();
      bf16* krow = dqkv + ((size_t)(row_base + kb * BKEY + r)) * 3 * C + C + h * HD + hf * NO;
      bf16* vrow = krow + C;
      float v[NO];
      if (NO == 32) tmem_ld32(tmem + lane_off + C_DK + hf * NO, *reinterpret_cast<float(*)[32]>(v));
      else tmem_ld16(tmem + lane_off + C_DK + hf * NO, *reinterpret_cast<float(*)[16]>(v));
#pragma unroll
      for (int i2 = 0; i2 < NO; i2 += 8)
        *reinterpret_cast<uint4*>(krow + i2) =
            make_uint4(pack_bf16x2(v[i2], v[i2 + 1]), pack_bf16x2(v[i2 + 2], v[i2 + 3]),
                       pack_bf16x2(v[i2 + 4], v[i2 + 5]), pack_bf16x2(v[i2 + 6], v[i2 + 7]));
      if (NO == 32) tmem_ld32(tmem + lane_off + C_DV + hf * NO, *reinterpret_cast<float(*)[32]>(v));
      else tmem_ld16(tmem + lane_off + C_DV + hf * NO, *reinterpret_cast<float(*)[16]>(v));
#pragma unroll
      for (int i2 = 0; i2 < NO; i2 += 8)
        *reinterpret_cast<uint4*>(vrow + i2) =
            make_uint4(pack_bf16x2(v[i2], v[i2 + 1]), pack_bf16x2(v[i2 + 2], v[i2 + 3]),
                       pack_bf16x2(v[i2 + 4], v[i2 + 5]), pack_bf16x2(v[i2 + 6], v[i2 + 7]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(dkdv_empty));
    }
    if (ok && g > 0) ok = drain_dq(g - 1, prev_hc, prev_qrow0);
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS_BWD);
  }
}

// The whole backward. xtiles (B*H*T*32 bytes) and dq_acc fp32 [B*T, C] are
// scratch (contents on entry do not matter); dqkv receives dQ | dK | dV. With
// dbias (fp32 [3C], 16-byte aligned) the gradient of the qkv bias is added
// there: column sums of dQ (post pass) and of dO (prep pass, the value third);
// the key third gets nothing, its gradient being exactly zero (adding one
// vector to every key shifts each query's scores by a constant, which the
// softmax removes).
template <int D>
static cudaError_t bwd_run(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, uint8_t* xtiles,
                           float* dq_acc, bf16* dqkv, float* dbias, int B, int T, int H, int* err,
                           cudaStream_t s) {
  using G = bwd::Geom<D>;
  static PerDeviceOnce once;
  cudaError_t e0 = once.run([] {
    // The register hand-over inside the kernel needs the block to be launched
    // with kLaunchRegs registers a thread; anything less would stall it.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_bwd_tc_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != bwd::kLaunchRegs) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(attn_bwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
  });
  if (e0 != cudaSuccess) return e0;
  if (H > bwd::kMaxHeads || T % bwd::kPrepRows || T % bwd::BKEY) return cudaErrorInvalidValue;
  const int C = H * D;
  const float scale = 1.0f / sqrtf((float)D);
  const CUtensorMapSwizzle swz = D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap tm_qkv, tm_do, tm_dq;
  // dQ boxes: 32 query rows x D/2 fp32 columns (128- or 64-byte rows)
  if (!encode_map_2d(&tm_qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, 3 * (uint64_t)C, (uint64_t)B * T,
                     3 * (uint64_t)C, D, 128, swz) ||
      !encode_map_2d(&tm_do, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dout, (uint64_t)C, (uint64_t)B * T, (uint64_t)C, D,
                     128, swz) ||
      !encode_map_2d(&tm_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dq_acc, (uint64_t)C, (uint64_t)B * T, (uint64_t)C,
                     D / 2, 32, swz))
    return cudaErrorInvalidValue;
  if (dbias && (reinterpret_cast<uintptr_t>(dbias) & 15)) return cudaErrorInvalidValue;
  // prep pass: ceil(C/256) warps per row group, as many row groups as fit 384 threads
  const int ng = (C / 8 + 31) / 32;
  const int prep_threads = 32 * ng * std::max(1, 12 / ng);
  launch_pdl(bwd_prep_kernel<D>, dim3(B * T / bwd::kPrepRows), dim3(prep_threads), 0, s, out, dout, lse, xtiles,
             dq_acc, dbias ? dbias + 2 * C : nullptr, T, H, scale);
  const int n_items = (T / bwd::BKEY) * B * H;
  const int sms = device_sm_count();   // one persistent CTA per SM
  const int grid = n_items < sms ? n_items : sms;
  launch_pdl(attn_bwd_tc_kernel<D>, dim3(grid), dim3(bwd::kThreads), G::SMEM_BYTES, s, tm_qkv, tm_do, tm_dq, xtiles,
             dqkv, T, H, B * H, scale, err);
  // post pass: C/8 chunk columns times as many row lanes as fit 1024 threads
  // (C/8 <= 512); one wave of blocks
  const int nv = C / 8, rows = B * T;
  const int rl = 1024 / nv;
  const int bps = std::max(1, 2048 / (nv * rl));
  const int post_blocks = std::max(1, std::min(sms * bps, (rows + rl - 1) / rl));
  launch_pdl(bwd_post_kernel, dim3(post_blocks), dim3(nv * rl), 0, s, dq_acc, dqkv, dbias, rows, C);
  return cudaGetLastError();
}

}  // namespace attn_tc
