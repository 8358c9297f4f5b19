// gpt2step: the GPT-2 training step on one B200 behind a C ABI.
//
// The model lives entirely inside one caller-provided device arena: fp32
// master weights, gradients and Adam moments as flat arrays (16 parameter
// kinds, each 64-element aligned), a bf16 copy of the weights for the tensor
// cores, every activation the backward pass needs, the bf16 logits (reused in
// place for their gradient) and small workspaces. The library allocates no
// device memory of its own.
//
// Step ("Pretraining and adapting a language model on a dependency-free
// stack", §4.1 model, §4.3 optimisation and precision, §4.4 accumulation):
//   forward   embed -> L x [LN1 -> QKV -> causal attention -> proj (+res)
//             -> LN2 -> fc + GELU -> proj (+res)] -> LN_f -> tied head -> CE
//   backward  the same in reverse, weight gradients accumulated in fp32
//   update    global norm over all gradients / micro-steps, clip, AdamW
#include <limits.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/gpt2step.h"
#include "../../include/gpt2step_ops.h"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "gemm2sm.cuh"
#include "kernels.cuh"

namespace {

enum KindId {
  K_WTE = 0, K_WPE, K_LN1W, K_LN1B, K_QKVW, K_QKVB, K_ATTPROJW, K_ATTPROJB,
  K_LN2W, K_LN2B, K_FCW, K_FCB, K_FCPROJW, K_FCPROJB, K_LNFW, K_LNFB, NUM_KINDS
};

constexpr int kNormBlocks = 2 * 148;
constexpr int kLnBwdBlocks = 2 * 148;
constexpr int kMaxStrips = 256;
// grouped dgrad + wgrad launches of the backward: the four linear layers of a
// block and the tied lm_head; each gets a tile plan of at most kSchedInts ints
enum GroupId { G_MLP_PROJ = 0, G_MLP_FC, G_ATTN_PROJ, G_QKV, G_LM_HEAD, kNumGroups };
constexpr int kSchedInts = 16384;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Dims {
  int L, H, C, T, V, Vp, B, hd;
  long N;  // B * T
};

bool resolve(const gpt2_config* c, Dims* d) {
  if (!c) return false;
  d->L = c->n_layer; d->H = c->n_head; d->C = c->n_embd; d->T = c->seq_len;
  d->V = c->vocab_real; d->B = c->micro_batch;
  d->Vp = c->vocab_padded ? c->vocab_padded : (c->vocab_real + 127) / 128 * 128;
  if (d->L < 0 || d->H <= 0 || d->C <= 0 || d->T <= 0 || d->V <= 1 || d->B <= 0) return false;
  if (d->C % d->H) return false;
  d->hd = d->C / d->H;
  if (d->hd != 32 && d->hd != 64) return false;
  if (d->C % 128 || d->T % 64 || d->T > 4096 || d->Vp % 128 || d->Vp < d->V) return false;
  switch (d->C) {
    case 128: case 256: case 384: case 512: case 768: case 1024: case 1536: case 2048: break;
    default: return false;
  }
  d->N = (long)d->B * d->T;
  return true;
}

struct KindInfo {
  long n;            // element count of the kind (all layers)
  int rows, cols;    // per-layer matrix shape (cols = 0 for vectors)
  bool per_layer, decay;
};

// Flat parameter layout (the same for params, grads, Adam m, v and the bf16 copy):
//   region 0  [0, P1)   the 1-D parameters (LayerNorm gains and biases, linear
//                       biases), kind by kind, layers contiguous;
//   buckets   [P1, P)   the 2-D weights (decayed), grouped by when the backward
//                       pass finishes their gradients: one bucket per block from
//                       the last to the first ({mlp proj, mlp fc, attention proj,
//                       qkv} of that block), then {wpe, wte}. Each bucket is padded
//                       with zeros to a multiple of kBucketAlign elements, so that
//                       it splits into equal 64-element-aligned shards for any
//                       world size dividing 120.
constexpr long kBucketAlign = 64 * 120;

struct Layout {
  Dims d;
  KindInfo kind[NUM_KINDS];
  std::vector<long> off[NUM_KINDS];   // element offset of each (kind, layer) block
  std::vector<long> bucket_end;        // end of each bucket; bucket 0 starts at P1
  long P1;   // end of the 1-D region (multiple of 64)
  long P;    // flat length
  size_t params, grads, adam_m, adam_v, pbf;
  size_t resid, ln1, ln1_mean, ln1_rstd, qkv, atty, lse, resid_mid, ln2, ln2_mean, ln2_rstd, fch, fchg;
  size_t lnf, lnf_mean, lnf_rstd, logits, lse_part;
  size_t dresid, dln, d4c, dqkv, datty, dq_acc, attD;
  size_t norm_part, losses, scalars, eval_acc, err, tok, tgt, sched;
  size_t total;
};

// (max, sum) partials per logits row that the lm_head GEMM leaves: two per 256-wide tile
inline int lse_slots(int Vp) { return 2 * ((Vp + 255) / 256); }

void make_layout(const Dims& d, Layout* lay) {
  lay->d = d;
  const long L = d.L, C = d.C;
  struct Def { int rows, cols; bool per_layer, decay; };
  const Def defs[NUM_KINDS] = {
      {d.Vp, d.C, false, true},  {d.T, d.C, false, true},  {d.C, 0, true, false},     {d.C, 0, true, false},
      {3 * d.C, d.C, true, true}, {3 * d.C, 0, true, false}, {d.C, d.C, true, true},   {d.C, 0, true, false},
      {d.C, 0, true, false},     {d.C, 0, true, false},     {4 * d.C, d.C, true, true}, {4 * d.C, 0, true, false},
      {d.C, 4 * d.C, true, true}, {d.C, 0, true, false},    {d.C, 0, false, false},    {d.C, 0, false, false}};
  for (int k = 0; k < NUM_KINDS; ++k) {
    const Def& f = defs[k];
    const long per = (long)f.rows * (f.cols ? f.cols : 1);
    lay->kind[k] = {per * (f.per_layer ? L : 1), f.rows, f.cols, f.per_layer, f.decay};
    lay->off[k].assign(f.per_layer ? (size_t)std::max<long>(L, 1) : 1, 0);
  }
  auto per = [&](int k) { return (long)lay->kind[k].rows * (lay->kind[k].cols ? lay->kind[k].cols : 1); };
  long off = 0;
  // region 0: the 1-D kinds
  const int vec_kinds[] = {K_LN1W, K_LN1B, K_QKVB, K_ATTPROJB, K_LN2W, K_LN2B, K_FCB, K_FCPROJB, K_LNFW, K_LNFB};
  for (int k : vec_kinds) {
    const int nl = lay->kind[k].per_layer ? (int)L : 1;
    for (int l = 0; l < nl; ++l) lay->off[k][l] = off + (long)l * per(k);
    off = (long)align_up(off + lay->kind[k].n, 64);
  }
  lay->P1 = off;
  // buckets of 2-D weights in the order the backward pass completes them
  lay->bucket_end.clear();
  for (int l = (int)L - 1; l >= 0; --l) {
    for (int k : {K_FCPROJW, K_FCW, K_ATTPROJW, K_QKVW}) {
      lay->off[k][l] = off;
      off += per(k);
    }
    off = (long)align_up(off, kBucketAlign);
    lay->bucket_end.push_back(off);
  }
  for (int k : {K_WPE, K_WTE}) {
    lay->off[k][0] = off;
    off += per(k);
  }
  off = (long)align_up(off, kBucketAlign);
  lay->bucket_end.push_back(off);
  lay->P = off;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes, 1024); return r; };
  const size_t P = (size_t)lay->P, N = (size_t)d.N;
  lay->params = take(P * 4);
  lay->grads = take(P * 4);
  lay->adam_m = take(P * 4);
  lay->adam_v = take(P * 4);
  lay->pbf = take(P * 2);
  lay->resid = take((L + 1) * N * C * 2);
  lay->ln1 = take(L * N * C * 2);
  lay->ln1_mean = take(L * N * 4);
  lay->ln1_rstd = take(L * N * 4);
  lay->qkv = take(L * N * 3 * C * 2);
  lay->atty = take(L * N * C * 2);
  lay->lse = take(L * N * d.H * 4);
  lay->resid_mid = take(L * N * C * 2);
  lay->ln2 = take(L * N * C * 2);
  lay->ln2_mean = take(L * N * 4);
  lay->ln2_rstd = take(L * N * 4);
  lay->fch = take(L * N * 4 * C * 2);
  lay->fchg = take(L * N * 4 * C * 2);
  lay->lnf = take(N * C * 2);
  lay->lnf_mean = take(N * 4);
  lay->lnf_rstd = take(N * 4);
  lay->logits = take(N * (size_t)d.Vp * 2);
  lay->lse_part = take(N * (size_t)lse_slots(d.Vp) * 8);
  lay->dresid = take(N * C * 2);
  lay->dln = take(N * C * 2);
  lay->d4c = take(N * 4 * C * 2);
  lay->dqkv = take(N * 3 * C * 2);
  lay->datty = take(N * C * 2);
  lay->dq_acc = take(N * C * 4);
  lay->attD = take(N * d.H * 32);
  lay->norm_part = take(kNormBlocks * 8);
  lay->sched = take((size_t)kNumGroups * kSchedInts * 4);
  lay->losses = take(N * 4);
  lay->scalars = take(sizeof(k::StepScalars));
  lay->eval_acc = take(64);
  lay->err = take(64);
  lay->tok = take(N * 4);
  lay->tgt = take(N * 4);
  lay->total = o;
}

const char* kind_layer_suffix(int k) {
  switch (k) {
    case K_LN1W: return "ln_1.weight";
    case K_LN1B: return "ln_1.bias";
    case K_QKVW: return "attn.c_attn.weight";
    case K_QKVB: return "attn.c_attn.bias";
    case K_ATTPROJW: return "attn.c_proj.weight";
    case K_ATTPROJB: return "attn.c_proj.bias";
    case K_LN2W: return "ln_2.weight";
    case K_LN2B: return "ln_2.bias";
    case K_FCW: return "mlp.c_fc.weight";
    case K_FCB: return "mlp.c_fc.bias";
    case K_FCPROJW: return "mlp.c_proj.weight";
    case K_FCPROJB: return "mlp.c_proj.bias";
    default: return "";
  }
}

}  // namespace

struct NamedTensor {
  std::string name;
  int kind, layer;
  long off, n;
  int64_t shape[2];
  int ndim;
};

// Optional per-class timing of the library's own launches with CUDA events on
// the model's stream (enabled by gpt2_profile_enable).
enum ProfClass { PC_GEMM = 0, PC_ATTN_FWD, PC_ATTN_BWD, PC_LN_FWD, PC_LN_BWD, PC_CE, PC_EMBED, PC_BIAS, PC_OPT, PC_N };
static const char* kProfNames[PC_N] = {"gemm", "attention_fwd", "attention_bwd", "layernorm_fwd", "layernorm_bwd",
                                       "softmax_ce", "embedding", "bias_grad", "clip_adamw"};

struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> ev;
  size_t used = 0;
  struct Entry { int cls; double work; size_t ev; };
  std::vector<Entry> pending;
  double ms[PC_N] = {}, work[PC_N] = {};
  int64_t n[PC_N] = {};
};

struct gpt2_model {
  gpt2_config cfg;
  Layout lay;
  cudaStream_t stream;
  char* arena;
  int n_micro;
  bool stepped;  // at least one clip_adamw has run
  int64_t launches = 0;  // kernels this model has launched
  Profiler prof;
  std::vector<cudaEvent_t> bucket_events;  // caller's events, recorded when each bucket's gradients are final
  int group_splits[kNumGroups] = {};       // planned wgrad splits (0: no plan for that group)
  std::vector<NamedTensor> tensors;
  ~gpt2_model() {
    for (cudaEvent_t e : prof.ev) cudaEventDestroy(e);
  }

  template <typename T>
  T* at(size_t off) const { return reinterpret_cast<T*>(arena + off); }
  float* params() const { return at<float>(lay.params); }
  float* grads() const { return at<float>(lay.grads); }
  bf16* pbf() const { return at<bf16>(lay.pbf); }
  long off(int k, int l) const { return lay.off[k][lay.kind[k].per_layer ? l : 0]; }
  float* P(int k, int l = 0) const { return params() + off(k, l); }
  float* G(int k, int l = 0) const { return grads() + off(k, l); }
  bf16* W(int k, int l = 0) const { return pbf() + off(k, l); }
  long per(int k) const { return (long)lay.kind[k].rows * (lay.kind[k].cols ? lay.kind[k].cols : 1); }
  int* err() const { return at<int>(lay.err); }
  k::StepScalars* sc() const { return at<k::StepScalars>(lay.scalars); }
};

// ---------------------------------------------------------------------------
// kernel launch helpers (shared by the model and the op-level entry points)
// ---------------------------------------------------------------------------
namespace launch {

// Resident CTAs of `kern` on the current device (blocks of `threads`, no dynamic shared memory).
template <typename K>
int resident_ctas(PerDeviceOnce& once, int (&cache)[PerDeviceOnce::kMaxDevices], K* kern, int threads) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= PerDeviceOnce::kMaxDevices) return 148;
  once.run([&] {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    cache[dev] = per_sm * device_sm_count();
    return cudaSuccess;
  });
  return cache[dev] > 0 ? cache[dev] : 148;
}

template <int C>
void ln_fwd_c(const bf16* x, const float* w, const float* b, bf16* y, float* mean, float* rstd, int rows,
              cudaStream_t s) {
  static PerDeviceOnce once;
  static int cache[PerDeviceOnce::kMaxDevices] = {};
  const int full = resident_ctas(once, cache, k::layernorm_fwd_kernel<C>, k::kLnFwdWarps * 32);
  const int per_cta = k::kLnFwdWarps * k::ln_fwd_rows(C);   // rows a CTA takes per pass
  const int need = (rows + per_cta - 1) / per_cta;
  launch_pdl(k::layernorm_fwd_kernel<C>, dim3(std::min(need, full)), dim3(k::kLnFwdWarps * 32), 0, s, x, w, b, y,
             mean, rstd, rows);
}

int ln_fwd(const bf16* x, const float* w, const float* b, bf16* y, float* mean, float* rstd, int rows, int C,
           cudaStream_t s) {
  switch (C) {
    case 128: ln_fwd_c<128>(x, w, b, y, mean, rstd, rows, s); break;
    case 256: ln_fwd_c<256>(x, w, b, y, mean, rstd, rows, s); break;
    case 384: ln_fwd_c<384>(x, w, b, y, mean, rstd, rows, s); break;
    case 512: ln_fwd_c<512>(x, w, b, y, mean, rstd, rows, s); break;
    case 768: ln_fwd_c<768>(x, w, b, y, mean, rstd, rows, s); break;
    case 1024: ln_fwd_c<1024>(x, w, b, y, mean, rstd, rows, s); break;
    case 1536: ln_fwd_c<1536>(x, w, b, y, mean, rstd, rows, s); break;
    case 2048: ln_fwd_c<2048>(x, w, b, y, mean, rstd, rows, s); break;
    default: return GPT2_ERR_ARG;
  }
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

int ln_bwd_blocks(int rows, int C) {
  const int warps = k::ln_bwd_warps(C);
  return std::min(148 * k::ln_bwd_minb(C), (rows + warps - 1) / warps);
}
static_assert(148 * 2 <= kLnBwdBlocks, "LayerNorm partial rows");

// Workspace of the LayerNorm backward: one partial row of nq * C floats per CTA
// (nq = 2: dw, db; nq = 3 adds the column sum of dx).
size_t ln_bwd_workspace(int rows, int C, int nq = 2) { return (size_t)ln_bwd_blocks(rows, C) * nq * C * 4; }

template <int C>
cudaError_t ln_bwd_c(const bf16* dy, const bf16* x, const float* mean, const float* rstd, const float* w,
                     const bf16* dresid, bf16* dx, float* part, int rows, int blocks, int with_dxsum, float* dw,
                     float* db, float* dbias, cudaStream_t s) {
  using Cfg = k::LnBwdCfg<C>;
  static PerDeviceOnce once;
  const cudaError_t e = smem_optin(once, k::layernorm_bwd_kernel<C>, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  launch_pdl(k::layernorm_bwd_kernel<C>, dim3(blocks), dim3(Cfg::WARPS * 32), Cfg::SMEM, s, dy, x, mean, rstd, w,
             dresid, dx, part, rows, with_dxsum, dw, db, dbias);
  return cudaGetLastError();
}

// dbias (may be NULL) receives the column sum of dx: the bias gradient of the
// projection whose output gradient dx is. With a workspace (`part`) the column
// sums are combined in a fixed order by a second launch (deterministic); with
// part == NULL each CTA adds its sums into dw, db, dbias by fp32 vector atomics
// in the same launch (dw, db, dbias then 16-byte aligned).
int ln_bwd(const bf16* dy, const bf16* x, const float* mean, const float* rstd, const float* w, const bf16* dresid,
           bf16* dx, float* dw, float* db, float* dbias, int rows, int C, float* part, size_t part_bytes,
           cudaStream_t s) {
  const int nq = dbias ? 3 : 2;
  const int blocks = ln_bwd_blocks(rows, C);
  if (part && part_bytes < (size_t)blocks * nq * C * 4) return GPT2_ERR_ARG;
  if (!part && ((reinterpret_cast<uintptr_t>(dw) | reinterpret_cast<uintptr_t>(db) |
                 reinterpret_cast<uintptr_t>(dbias)) & 15))
    return GPT2_ERR_ARG;
  const int wd = dbias ? 1 : 0;
  cudaError_t e;
  switch (C) {
#define GPT2_LN_BWD_CASE(CC) \
    case CC: e = ln_bwd_c<CC>(dy, x, mean, rstd, w, dresid, dx, part, rows, blocks, wd, dw, db, dbias, s); break;
    GPT2_LN_BWD_CASE(128) GPT2_LN_BWD_CASE(256) GPT2_LN_BWD_CASE(384) GPT2_LN_BWD_CASE(512)
    GPT2_LN_BWD_CASE(768) GPT2_LN_BWD_CASE(1024) GPT2_LN_BWD_CASE(1536) GPT2_LN_BWD_CASE(2048)
#undef GPT2_LN_BWD_CASE
    default: return GPT2_ERR_ARG;
  }
  if (e != cudaSuccess) return GPT2_ERR_CUDA;
  if (part)
    launch_pdl(k::partial_rows_reduce_kernel, dim3((nq * C + 31) / 32), dim3(256), 0, s, part, blocks, nq * C, dw, db,
               dbias, C);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

void colsum_geometry(int M, int N, int* strips, int* rows_per_strip) {
  const int gx = (N / 8 + 31) / 32;
  int st = std::max(1, 4 * 148 / gx);
  st = std::min(st, std::max(1, (M + 63) / 64));
  st = std::min(st, kMaxStrips);
  *rows_per_strip = (M + st - 1) / st;
  *strips = (M + *rows_per_strip - 1) / *rows_per_strip;
}

size_t bias_grad_workspace(int M, int N) {
  int strips, rps;
  colsum_geometry(M, N, &strips, &rps);
  return (size_t)strips * N * 4;
}

// With a workspace the strips' sums are combined in a fixed order by a second
// launch (deterministic); with part == NULL they go into db by fp32 atomics in
// the same launch (db then 16-byte aligned).
int bias_grad(const bf16* dout, float* db, int M, int N, float* part, size_t part_bytes, cudaStream_t s) {
  if (N % 8) return GPT2_ERR_ARG;
  int strips, rps;
  colsum_geometry(M, N, &strips, &rps);
  if (part && part_bytes < (size_t)strips * N * 4) return GPT2_ERR_ARG;
  if (!part && (reinterpret_cast<uintptr_t>(db) & 15)) return GPT2_ERR_ARG;
  dim3 grid((N / 8 + 31) / 32, strips);
  launch_pdl(k::colsum_partial_kernel, dim3(grid), dim3(256), 0, s, dout, part, M, N, rps, db);
  if (part) launch_pdl(k::colsum_final_kernel, dim3((N + 255) / 256), dim3(256), 0, s, part, db, strips, N);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

// ignore_index: targets equal to it are skipped (INT_MIN: none are). part: the
// logits GEMM's EPI_LSE row partials ([N][slots]), or null to scan the row.
int softmax_ce(bf16* logits, const int32_t* targets, float* losses, int N, int V, int Vp, float dscale,
               int write_grad, int* err, cudaStream_t s, int ignore_index = INT_MIN,
               const float2* part = nullptr, int slots = 0, const float* tgt_val = nullptr) {
  if (Vp % 8 || V > Vp || V <= 0) return GPT2_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(logits) & 15) != 0) return GPT2_ERR_ARG;
  if (part && slots <= 0) return GPT2_ERR_ARG;
  if (tgt_val && (!part || write_grad)) return GPT2_ERR_ARG;   // logits-free: a loss from the partials only
  if (!logits && !tgt_val) return GPT2_ERR_ARG;
  launch_pdl(k::softmax_ce_kernel, dim3(N), dim3(k::kCeThreads), 0, s, logits, targets, losses, V, Vp, dscale,
             write_grad, err, ignore_index, part, slots, tgt_val);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

// Head size 64 with T a multiple of 128 runs on tcgen05 (S, O in tensor memory);
// other supported shapes use the mma.sync kernel.
int attention_fwd(const bf16* qkv, bf16* out, float* lse, int B, int T, int H, int hd, int* err, cudaStream_t s) {
  if (T % 64) return GPT2_ERR_ARG;
  cudaError_t e;
  if (hd == 64 && T % attn_tc::BQ == 0 && err != nullptr) e = attn_tc::fwd<64>(qkv, out, lse, B, T, H, err, s);
  else if (hd == 32 && T % attn_tc::BQ == 0 && err != nullptr) e = attn_tc::fwd<32>(qkv, out, lse, B, T, H, err, s);
  else if (hd == 64) e = attn::fwd<64>(qkv, out, lse, B, T, H, s);
  else if (hd == 32) e = attn::fwd<32>(qkv, out, lse, B, T, H, s);
  else return GPT2_ERR_ARG;
  return e == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

// dbias (fp32 [3C], or null): += the gradient of the qkv bias. On tcgen05 the
// attention backward's own passes add it (the key third exactly zero); on the
// mma.sync path the column sums of the stored dqkv are added afterwards.
int attention_bwd(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, float* Dv, float* dq_acc,
                  bf16* dqkv, float* dbias, int B, int T, int H, int hd, int* err, cudaStream_t s) {
  if (T % 64) return GPT2_ERR_ARG;
  if (dbias && (reinterpret_cast<uintptr_t>(dbias) & 15)) return GPT2_ERR_ARG;
  cudaError_t e;
  if ((hd == 64 || hd == 32) && T % attn_tc::bwd::BKEY == 0 && H <= attn_tc::bwd::kMaxHeads && err != nullptr) {
    // Dv holds the 16-column per-query operand tiles here (32 bytes per query and head)
    uint8_t* xt = reinterpret_cast<uint8_t*>(Dv);
    e = hd == 64 ? attn_tc::bwd_run<64>(qkv, out, dout, lse, xt, dq_acc, dqkv, dbias, B, T, H, err, s)
                 : attn_tc::bwd_run<32>(qkv, out, dout, lse, xt, dq_acc, dqkv, dbias, B, T, H, err, s);
    return e == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
  }
  if (hd == 64) e = attn::bwd<64>(qkv, out, dout, lse, Dv, dq_acc, dqkv, B, T, H, s);
  else if (hd == 32) e = attn::bwd<32>(qkv, out, dout, lse, Dv, dq_acc, dqkv, B, T, H, s);
  else return GPT2_ERR_ARG;
  if (e != cudaSuccess) return GPT2_ERR_CUDA;
  return dbias ? bias_grad(dqkv, dbias, B * T, 3 * H * hd, nullptr, 0, s) : GPT2_OK;
}

int grid_for(long work, int threads) {
  long b = (work + threads - 1) / threads;
  if (b > 148L * 16) b = 148L * 16;
  if (b < 1) b = 1;
  return (int)b;
}

}  // namespace launch

// ---------------------------------------------------------------------------
// the model's forward / backward sequences
// ---------------------------------------------------------------------------
namespace {

#define GPT2_TRY(x)                 \
  do {                              \
    int _st = (x);                  \
    if (_st != GPT2_OK) return _st; \
  } while (0)

gemm::Call gemm_call(gemm::Kind kind, int epi, int M, int N, int K, int* err) {
  gemm::Call c{};
  c.kind = kind; c.epi = epi; c.M = M; c.N = N; c.K = K; c.err = err;
  return c;
}

// Begin / end one profiled launch group; `nlaunch` kernels are counted either way.
size_t prof_begin(gpt2_model* m) {
  Profiler& p = m->prof;
  if (!p.on) return SIZE_MAX;
  while (p.ev.size() < p.used + 2) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return SIZE_MAX;
    p.ev.push_back(e);
  }
  const size_t i = p.used;
  p.used += 2;
  cudaEventRecord(p.ev[i], m->stream);
  return i;
}

void prof_end(gpt2_model* m, size_t i, int cls, double work, int nlaunch) {
  m->launches += nlaunch;
  if (i == SIZE_MAX) return;
  cudaEventRecord(m->prof.ev[i + 1], m->stream);
  m->prof.pending.push_back({cls, work, i});
}

int run_gemm(gpt2_model* m, const gemm::Call& c) {
  const size_t p = prof_begin(m);
  const int st = gemm2::run(c, m->stream);
  prof_end(m, p, PC_GEMM, 2.0 * c.M * c.N * c.K, 1);
  return st;
}

// A layer's dgrad (c0) and wgrad (c1) as one grouped launch where possible, on
// the tile plan made at creation for that group.
int run_gemm_group(gpt2_model* m, const gemm::Call& c0, const gemm::Call& c1, int group) {
  const size_t p = prof_begin(m);
  int nl = 2;
  const int sp = m->group_splits[group];
  const int* sched = sp ? m->at<int>(m->lay.sched) + (size_t)group * kSchedInts : nullptr;
  const int st = gemm2::run_group(c0, c1, m->stream, &nl, nullptr, sp, sched);
  prof_end(m, p, PC_GEMM, 2.0 * c0.M * c0.N * c0.K + 2.0 * c1.M * c1.N * c1.K, nl);
  return st;
}

int ln_fwd_m(gpt2_model* m, const bf16* x, int kw, int kb, int l, bf16* y, float* mean, float* rstd, int rows) {
  const int C = m->lay.d.C;
  const size_t p = prof_begin(m);
  const int st = launch::ln_fwd(x, m->P(kw, l), m->P(kb, l), y, mean, rstd, rows, C, m->stream);
  prof_end(m, p, PC_LN_FWD, (double)rows * (4.0 * C + 8), 1);
  return st;
}

// Forward over `b` sequences; `train` keeps dlogits for the backward pass,
// otherwise only losses are produced. Loss sum goes to *loss_acc.
int forward(gpt2_model* m, const int32_t* tok, const int32_t* tgt, int b, bool train, double* loss_acc) {
  const Layout& y = m->lay;
  const Dims& d = y.d;
  const int C = d.C, T = d.T, L = d.L;
  const long N = (long)b * T;
  const size_t NC = (size_t)d.N * C;  // per-layer stride of the saved activations
  cudaStream_t s = m->stream;
  int* err = m->err();
  bf16* resid = m->at<bf16>(y.resid);

  {
    const size_t p = prof_begin(m);
    launch_pdl(k::embed_fwd_kernel, dim3(launch::grid_for(N * C / 8, 256)), dim3(256), 0, s, tok, m->W(K_WTE),
               m->W(K_WPE), resid, (int)N, T, C, d.V, err);
    prof_end(m, p, PC_EMBED, (double)N * (6.0 * C + 4), 1);
  }
  for (int l = 0; l < L; ++l) {
    bf16* x_in = resid + l * NC;
    bf16* ln1 = m->at<bf16>(y.ln1) + l * NC;
    bf16* qkv = m->at<bf16>(y.qkv) + l * NC * 3;
    bf16* atty = m->at<bf16>(y.atty) + l * NC;
    bf16* xmid = m->at<bf16>(y.resid_mid) + l * NC;
    bf16* ln2 = m->at<bf16>(y.ln2) + l * NC;
    bf16* fch = m->at<bf16>(y.fch) + l * NC * 4;
    bf16* fchg = m->at<bf16>(y.fchg) + l * NC * 4;
    float* lse = m->at<float>(y.lse) + (size_t)l * d.N * d.H;
    GPT2_TRY(ln_fwd_m(m, x_in, K_LN1W, K_LN1B, l, ln1, m->at<float>(y.ln1_mean) + l * d.N,
                      m->at<float>(y.ln1_rstd) + l * d.N, (int)N));
    {
      gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_STORE, (int)N, 3 * C, C, err);
      c.a = ln1; c.lda = C; c.b = m->W(K_QKVW, l); c.ldb = C; c.out = qkv; c.ldo = 3 * C; c.bias = m->P(K_QKVB, l);
      GPT2_TRY(run_gemm(m, c));
    }
    {
      const size_t p = prof_begin(m);
      GPT2_TRY(launch::attention_fwd(qkv, atty, lse, b, T, d.H, d.hd, err, s));
      // causal FLOPs: QK^T and PV over the T(T+1)/2 visible (query, key) pairs
      prof_end(m, p, PC_ATTN_FWD, 2.0 * b * d.H * (double)T * (T + 1) * d.hd, 1);
    }
    {
      gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_RESID, (int)N, C, C, err);
      c.a = atty; c.lda = C; c.b = m->W(K_ATTPROJW, l); c.ldb = C; c.out = xmid; c.ldo = C;
      c.bias = m->P(K_ATTPROJB, l); c.aux = x_in; c.ld_aux = C;
      GPT2_TRY(run_gemm(m, c));
    }
    GPT2_TRY(ln_fwd_m(m, xmid, K_LN2W, K_LN2B, l, ln2, m->at<float>(y.ln2_mean) + l * d.N,
                      m->at<float>(y.ln2_rstd) + l * d.N, (int)N));
    {
      // on CTA pairs the fc epilogue saves GELU'(x) for the backward instead of x
      // (one tanh for both outputs; the backward's epilogue is then one multiply)
      gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_GELU, (int)N, 4 * C, C, err);
      c.a = ln2; c.lda = C; c.b = m->W(K_FCW, l); c.ldb = C; c.out = fch; c.out2 = fchg; c.ldo = 4 * C;
      c.bias = m->P(K_FCB, l);
      if (gemm2::uses_pair(c)) c.epi = gemm::EPI_GELU_D;
      GPT2_TRY(run_gemm(m, c));
    }
    {
      gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_RESID, (int)N, C, 4 * C, err);
      c.a = fchg; c.lda = 4 * C; c.b = m->W(K_FCPROJW, l); c.ldb = 4 * C; c.out = resid + (l + 1) * NC; c.ldo = C;
      c.bias = m->P(K_FCPROJB, l); c.aux = xmid; c.ld_aux = C;
      GPT2_TRY(run_gemm(m, c));
    }
  }
  bf16* lnf = m->at<bf16>(y.lnf);
  GPT2_TRY(ln_fwd_m(m, resid + L * NC, K_LNFW, K_LNFB, 0, lnf, m->at<float>(y.lnf_mean), m->at<float>(y.lnf_rstd),
                    (int)N));
  bf16* logits = m->at<bf16>(y.logits);
  float* losses = m->at<float>(y.losses);
  // the pair kernel's epilogue also leaves each row's (max, sum) partials, so the
  // cross-entropy reads the logits once; for a loss alone (evaluation) it keeps
  // only the partials and the target logit, and the logits are never stored
  float2* lse_part = nullptr;
  bool logits_free = false;
  {
    gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_STORE, (int)N, d.Vp, C, err);
    c.a = lnf; c.lda = C; c.b = m->W(K_WTE); c.ldb = C; c.out = logits; c.ldo = d.Vp;
    if (gemm2::uses_pair(c)) {
      lse_part = m->at<float2>(y.lse_part);
      c.epi = gemm::EPI_LSE; c.lse_part = lse_part; c.lse_V = d.V;
      if (!train) {
        c.epi = gemm::EPI_LSE_ONLY; c.lse_tgt = tgt; c.lse_tgt_val = losses;
        logits_free = true;
      }
    }
    GPT2_TRY(run_gemm(m, c));
  }
  {
    const size_t p = prof_begin(m);
    GPT2_TRY(launch::softmax_ce(logits_free ? nullptr : logits, tgt, losses, (int)N, d.V, d.Vp, 1.0f / (float)N,
                                train ? 1 : 0, err, s, INT_MIN, lse_part, lse_slots(d.Vp),
                                logits_free ? losses : nullptr));
    launch_pdl(k::loss_reduce_kernel, dim3(1), dim3(1024), 0, s, losses, (int)N, loss_acc, &m->sc()->micro_loss);
    // algorithmic bytes: the logits read (and overwritten when training), or with
    // the GEMM's partials those plus the partials, and no row scan for a loss alone
    const double part_bytes = lse_part ? (double)N * lse_slots(d.Vp) * 8.0 : 0.0;
    const double row_bytes = train ? 4.0 * d.Vp : (lse_part ? 2.0 : 2.0 * d.Vp);
    prof_end(m, p, PC_CE, (double)N * row_bytes + part_bytes, 2);
  }
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

int bias_grad_m(gpt2_model* m, const bf16* dout, float* db, int M, int N) {
  const size_t p = prof_begin(m);
  const int st = launch::bias_grad(dout, db, M, N, nullptr, 0, m->stream);
  prof_end(m, p, PC_BIAS, 2.0 * M * N, 1);
  return st;
}

int ln_bwd_m(gpt2_model* m, const bf16* dy, const bf16* x, const float* mean, const float* rstd, int kw, int kb,
             int l, const bf16* dresid, bf16* dx, float* dbias) {
  const Dims& d = m->lay.d;
  const size_t p = prof_begin(m);
  const int st = launch::ln_bwd(dy, x, mean, rstd, m->P(kw, l), dresid, dx, m->G(kw, l), m->G(kb, l), dbias,
                                (int)d.N, d.C, nullptr, 0, m->stream);
  prof_end(m, p, PC_LN_BWD, (double)d.N * ((dresid ? 8.0 : 6.0) * d.C + 8), 1);
  return st;
}

int backward(gpt2_model* m, const int32_t* tok) {
  const Layout& y = m->lay;
  const Dims& d = y.d;
  const int C = d.C, T = d.T, L = d.L;
  const int N = (int)d.N;
  const size_t NC = (size_t)d.N * C;
  cudaStream_t s = m->stream;
  int* err = m->err();
  bf16* resid = m->at<bf16>(y.resid);
  bf16* dresid = m->at<bf16>(y.dresid);
  bf16* dln = m->at<bf16>(y.dln);
  bf16* d4c = m->at<bf16>(y.d4c);
  bf16* dqkv = m->at<bf16>(y.dqkv);
  bf16* datty = m->at<bf16>(y.datty);
  bf16* dlogits = m->at<bf16>(y.logits);
  bf16* lnf = m->at<bf16>(y.lnf);

  // tied head: dlnf = dlogits . wte ; dwte += dlogits^T . lnf (one grouped launch)
  {
    gemm::Call cd = gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, d.Vp, err);
    cd.a = dlogits; cd.lda = d.Vp; cd.b = m->W(K_WTE); cd.ldb = C; cd.out = dln; cd.ldo = C;
    gemm::Call cw = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, d.Vp, C, N, err);
    cw.a = dlogits; cw.lda = d.Vp; cw.b = lnf; cw.ldb = C; cw.outf = m->G(K_WTE); cw.ldf = C;
    GPT2_TRY(run_gemm_group(m, cd, cw, G_LM_HEAD));
  }
  // the residual gradient leaving ln_f is the output gradient of the last MLP projection
  GPT2_TRY(ln_bwd_m(m, dln, resid + L * NC, m->at<float>(y.lnf_mean), m->at<float>(y.lnf_rstd), K_LNFW, K_LNFB, 0,
                    nullptr, dresid, L > 0 ? m->G(K_FCPROJB, L - 1) : nullptr));

  for (int l = L - 1; l >= 0; --l) {
    bf16* x_in = resid + l * NC;
    bf16* ln1 = m->at<bf16>(y.ln1) + l * NC;
    bf16* qkv = m->at<bf16>(y.qkv) + l * NC * 3;
    bf16* atty = m->at<bf16>(y.atty) + l * NC;
    bf16* xmid = m->at<bf16>(y.resid_mid) + l * NC;
    bf16* ln2 = m->at<bf16>(y.ln2) + l * NC;
    bf16* fch = m->at<bf16>(y.fch) + l * NC * 4;
    bf16* fchg = m->at<bf16>(y.fchg) + l * NC * 4;
    float* lse = m->at<float>(y.lse) + (size_t)l * d.N * d.H;

    bool fused_fcb = false;   // fc bias gradient summed in the d4c epilogue
    // Each linear layer's input gradient (dgrad) and weight gradient (wgrad) run as
    // one grouped launch: the wgrad tiles fill the dgrad's last wave.
    // MLP projection (the GELU' epilogue also sums the fc bias gradient)
    {
      gemm::Call cw = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, C, 4 * C, N, err);
      cw.a = dresid; cw.lda = C; cw.b = fchg; cw.ldb = 4 * C; cw.outf = m->G(K_FCPROJW, l); cw.ldf = 4 * C;
      gemm::Call cd = gemm_call(gemm::DGRAD, gemm::EPI_DGELU, N, 4 * C, C, err);
      cd.a = dresid; cd.lda = C; cd.b = m->W(K_FCPROJW, l); cd.ldb = 4 * C; cd.out = d4c; cd.ldo = 4 * C;
      cd.aux = fch; cd.ld_aux = 4 * C;
      cd.colsum = m->G(K_FCB, l);
      fused_fcb = gemm2::uses_pair(cd);
      if (!fused_fcb) cd.colsum = nullptr;
      // the forward's fc epilogue saved GELU'(x) exactly when it ran on CTA pairs
      // (the same [N, 4C] output shape decides both)
      if (fused_fcb) cd.epi = gemm::EPI_DMUL;
      GPT2_TRY(run_gemm_group(m, cd, cw, G_MLP_PROJ));
    }
    // MLP fc
    {
      gemm::Call cw = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, 4 * C, C, N, err);
      cw.a = d4c; cw.lda = 4 * C; cw.b = ln2; cw.ldb = C; cw.outf = m->G(K_FCW, l); cw.ldf = C;
      gemm::Call cd = gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, 4 * C, err);
      cd.a = d4c; cd.lda = 4 * C; cd.b = m->W(K_FCW, l); cd.ldb = C; cd.out = dln; cd.ldo = C;
      GPT2_TRY(run_gemm_group(m, cd, cw, G_MLP_FC));
    }
    if (!fused_fcb) GPT2_TRY(bias_grad_m(m, d4c, m->G(K_FCB, l), N, 4 * C));
    GPT2_TRY(ln_bwd_m(m, dln, xmid, m->at<float>(y.ln2_mean) + l * d.N, m->at<float>(y.ln2_rstd) + l * d.N, K_LN2W,
                      K_LN2B, l, dresid, dresid, m->G(K_ATTPROJB, l)));
    // attention projection
    {
      gemm::Call cw = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, C, C, N, err);
      cw.a = dresid; cw.lda = C; cw.b = atty; cw.ldb = C; cw.outf = m->G(K_ATTPROJW, l); cw.ldf = C;
      gemm::Call cd = gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, C, err);
      cd.a = dresid; cd.lda = C; cd.b = m->W(K_ATTPROJW, l); cd.ldb = C; cd.out = datty; cd.ldo = C;
      GPT2_TRY(run_gemm_group(m, cd, cw, G_ATTN_PROJ));
    }
    {
      const size_t p = prof_begin(m);
      // the qkv bias gradient comes out of the attention backward's own passes
      GPT2_TRY(launch::attention_bwd(qkv, atty, datty, lse, m->at<float>(y.attD), m->at<float>(y.dq_acc), dqkv,
                                     m->G(K_QKVB, l), d.B, T, d.H, d.hd, err, s));
      // causal FLOPs: QK^T, dO V^T, dV, dK and dQ over the visible pairs
      prof_end(m, p, PC_ATTN_BWD, 5.0 * d.B * d.H * (double)T * (T + 1) * d.hd, 3);
    }
    // QKV projection
    {
      gemm::Call cw = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, 3 * C, C, N, err);
      cw.a = dqkv; cw.lda = 3 * C; cw.b = ln1; cw.ldb = C; cw.outf = m->G(K_QKVW, l); cw.ldf = C;
      gemm::Call cd = gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, 3 * C, err);
      cd.a = dqkv; cd.lda = 3 * C; cd.b = m->W(K_QKVW, l); cd.ldb = C; cd.out = dln; cd.ldo = C;
      GPT2_TRY(run_gemm_group(m, cd, cw, G_QKV));
    }
    // every 2-D weight gradient of this block is final for this micro-step
    if (!m->bucket_events.empty() && cudaEventRecord(m->bucket_events[L - 1 - l], s) != cudaSuccess)
      return GPT2_ERR_CUDA;
    GPT2_TRY(ln_bwd_m(m, dln, x_in, m->at<float>(y.ln1_mean) + l * d.N, m->at<float>(y.ln1_rstd) + l * d.N, K_LN1W,
                      K_LN1B, l, dresid, dresid, l > 0 ? m->G(K_FCPROJB, l - 1) : nullptr));
  }
  // embeddings
  {
    const size_t p = prof_begin(m);
    launch_pdl(k::embed_bwd_wpe_kernel, dim3((T * C / 8 + 255) / 256), dim3(256), 0, s, dresid, m->G(K_WPE), d.B, T, C);
    launch_pdl(k::embed_bwd_wte_kernel, dim3((N + k::kEmbRows - 1) / k::kEmbRows), dim3(256), 0, s, tok, dresid,
               m->G(K_WTE), N, C, d.V);
    prof_end(m, p, PC_EMBED, (double)N * (2.0 * C + 4) + 2.0 * N * C * 4 + 8.0 * T * C, 2);
  }
  // the last bucket (wpe, wte) and the 1-D region are final now
  if (!m->bucket_events.empty() && cudaEventRecord(m->bucket_events.back(), s) != cudaSuccess) return GPT2_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

// The status a device error word maps to (a timeout first: it means a kernel gave up early).
int status_of_device_word(int h) {
  if (h & DEVERR_TIMEOUT) return GPT2_ERR_TIMEOUT;
  if (h & DEVERR_TOKEN_RANGE) return GPT2_ERR_TOKEN_RANGE;
  if (h & DEVERR_NONFINITE) return GPT2_ERR_NONFINITE;
  return GPT2_OK;
}

// Tile plans of the backward's grouped launches (the shapes are fixed by the
// configuration), built on the host once and copied into the arena.
int make_group_plans(gpt2_model* m) {
  const Dims& d = m->lay.d;
  const int N = (int)d.N, C = d.C;
  struct Pair { gemm::Call cd, cw; };
  Pair g[kNumGroups] = {
      {gemm_call(gemm::DGRAD, gemm::EPI_DGELU, N, 4 * C, C, nullptr),
       gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, C, 4 * C, N, nullptr)},
      {gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, 4 * C, nullptr),
       gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, 4 * C, C, N, nullptr)},
      {gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, C, nullptr),
       gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, C, C, N, nullptr)},
      {gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, 3 * C, nullptr),
       gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, 3 * C, C, N, nullptr)},
      {gemm_call(gemm::DGRAD, gemm::EPI_STORE, N, C, d.Vp, nullptr),
       gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, d.Vp, C, N, nullptr)}};
  std::vector<int> host((size_t)kNumGroups * kSchedInts, 0);
  const int pairs = gemm::num_sms() / 2;
  for (int gi = 0; gi < kNumGroups; ++gi) {
    m->group_splits[gi] = 0;
    // The MLP projection's dgrad tiles carry the GELU' epilogue (the saved
    // pre-activation read, GELU', the fc bias column sums), which outlasts their
    // 12 k-blocks; the k-block cost model does not see that, and its plan measured
    // 11% slower than the static stride with the split the stride simulation picks.
    if (gi == G_MLP_PROJ) continue;
    if (!gemm2::groupable(g[gi].cd, g[gi].cw)) continue;
    const gemm2::GroupPlan plan = gemm2::plan_group(g[gi].cd, g[gi].cw, pairs);
    if (plan.splits1 <= 0 || plan.table.size() > (size_t)kSchedInts) continue;
    std::copy(plan.table.begin(), plan.table.end(), host.begin() + (size_t)gi * kSchedInts);
    m->group_splits[gi] = plan.splits1;
  }
  if (cudaMemcpyAsync(m->at<int>(m->lay.sched), host.data(), host.size() * sizeof(int), cudaMemcpyHostToDevice,
                      m->stream) != cudaSuccess ||
      cudaStreamSynchronize(m->stream) != cudaSuccess)
    return GPT2_ERR_CUDA;
  return GPT2_OK;
}

// Read and clear the device error word; map it to a status.
int collect_device_error(gpt2_model* m) {
  int h = 0;
  if (cudaMemcpyAsync(&h, m->err(), sizeof(int), cudaMemcpyDeviceToHost, m->stream) != cudaSuccess)
    return GPT2_ERR_CUDA;
  if (cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  if (h) {
    if (cudaMemsetAsync(m->err(), 0, sizeof(int), m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
    if (cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  }
  return status_of_device_word(h);
}

double lr_at(const gpt2_config& c, int step) {
  if (step < c.warmup_steps) return (double)c.max_lr * (step + 1) / c.warmup_steps;
  const int span = std::max(1, c.total_steps - c.warmup_steps);
  double ratio = (double)(step - c.warmup_steps) / span;
  if (ratio > 1.0) ratio = 1.0;
  const double coeff = 0.5 * (1.0 + cos(M_PI * ratio));
  return (double)c.min_lr + coeff * ((double)c.max_lr - (double)c.min_lr);
}

}  // namespace

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

size_t gpt2_arena_bytes(const gpt2_config* cfg) {
  Dims d;
  if (!resolve(cfg, &d)) return 0;
  Layout lay;
  make_layout(d, &lay);
  return lay.total;
}

int64_t gpt2_num_params(const gpt2_config* cfg, int padded) {
  Dims d;
  if (!resolve(cfg, &d)) return -1;
  Layout lay;
  make_layout(d, &lay);
  int64_t n = 0;
  for (int k = 0; k < NUM_KINDS; ++k) n += lay.kind[k].n;
  if (!padded) n -= (int64_t)(d.Vp - d.V) * d.C;
  return n;
}

const char* gpt2_status_string(int st) {
  switch (st) {
    case GPT2_OK: return "ok";
    case GPT2_ERR_ARG: return "invalid argument";
    case GPT2_ERR_CUDA: return "CUDA error";
    case GPT2_ERR_TOKEN_RANGE: return "token id out of range";
    case GPT2_ERR_NONFINITE: return "non-finite loss or gradient norm; step not applied";
    case GPT2_ERR_STATE: return "call out of order";
    case GPT2_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int gpt2_create(const gpt2_config* cfg, uint64_t seed, void* dev_arena, size_t arena_bytes, void* cuda_stream,
                gpt2_model** out) {
  if (!out) return GPT2_ERR_ARG;
  *out = nullptr;
  Dims d;
  if (!resolve(cfg, &d) || !dev_arena || (reinterpret_cast<uintptr_t>(dev_arena) & 1023)) return GPT2_ERR_ARG;
  gpt2_model* m = new gpt2_model();
  m->cfg = *cfg;
  m->cfg.vocab_padded = d.Vp;
  make_layout(d, &m->lay);
  if (arena_bytes < m->lay.total) { delete m; return GPT2_ERR_ARG; }
  m->arena = static_cast<char*>(dev_arena);
  m->stream = static_cast<cudaStream_t>(cuda_stream);
  m->n_micro = 0;
  m->stepped = false;
  // named tensors
  auto add = [&](const std::string& name, int kind, int layer) {
    NamedTensor t;
    t.name = name; t.kind = kind; t.layer = layer;
    const KindInfo& ki = m->lay.kind[kind];
    const long per = (long)ki.rows * (ki.cols ? ki.cols : 1);
    t.off = m->off(kind, layer > 0 ? layer : 0);
    t.n = per;
    t.ndim = ki.cols ? 2 : 1;
    t.shape[0] = ki.rows;
    t.shape[1] = ki.cols;
    m->tensors.push_back(t);
  };
  add("wte.weight", K_WTE, -1);
  add("wpe.weight", K_WPE, -1);
  for (int l = 0; l < d.L; ++l)
    for (int kk = K_LN1W; kk <= K_FCPROJB; ++kk) add("h." + std::to_string(l) + "." + kind_layer_suffix(kk), kk, l);
  add("ln_f.weight", K_LNFW, -1);
  add("ln_f.bias", K_LNFB, -1);

  cudaStream_t s = m->stream;
  // zero everything that accumulates (grads, moments, workspaces, scalars)
  if (cudaMemsetAsync(m->arena, 0, m->lay.total, s) != cudaSuccess) { delete m; return GPT2_ERR_CUDA; }
  const float proj_std = 0.02f / sqrtf(2.0f * (float)std::max(1, d.L));
  for (int kk = 0; kk < NUM_KINDS; ++kk) {
    const KindInfo& ki = m->lay.kind[kk];
    int mode;
    float sd = 0.f;
    long zero_from = ki.n;
    switch (kk) {
      case K_WTE: mode = 0; sd = 0.02f; zero_from = (long)d.V * d.C; break;
      case K_WPE: case K_QKVW: case K_FCW: mode = 0; sd = 0.02f; break;
      case K_ATTPROJW: case K_FCPROJW: mode = 0; sd = proj_std; break;
      case K_LN1W: case K_LN2W: case K_LNFW: mode = 1; break;
      default: mode = 2; break;
    }
    if (ki.n == 0) continue;
    // one launch per (kind, layer) block; the generator's counter runs over the
    // kind's elements in layer order, whatever the block's place in the layout
    const long per = m->per(kk);
    const int nl = ki.per_layer ? d.L : 1;
    for (int l = 0; l < nl; ++l) {
      const long o = m->off(kk, l);
      k::init_kind_kernel<<<launch::grid_for((per + 3) / 4, 256), 256, 0, s>>>(
          m->params() + o, m->pbf() + o, per, mode, sd, (uint32_t)kk, seed, zero_from, (long)l * per / 4);
    }
  }
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) { delete m; return GPT2_ERR_CUDA; }
  if (make_group_plans(m) != GPT2_OK) { delete m; return GPT2_ERR_CUDA; }
  *out = m;
  return GPT2_OK;
}

void gpt2_destroy(gpt2_model* m) { delete m; }

int gpt2_fwd_bwd(gpt2_model* m, const int32_t* tokens, const int32_t* targets, float* loss_out) {
  if (!m || !tokens || !targets) return GPT2_ERR_ARG;
  GPT2_TRY(forward(m, tokens, targets, m->lay.d.B, true, &m->sc()->loss_sum));
  GPT2_TRY(backward(m, tokens));
  m->n_micro += 1;
  if (loss_out) {
    GPT2_TRY(collect_device_error(m));
    if (cudaMemcpy(loss_out, &m->sc()->micro_loss, sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
      return GPT2_ERR_CUDA;
  }
  return GPT2_OK;
}

// Host-side form of element ranges: float4 ranges, validated against the layout
// (each 64-element aligned, inside [0, P), at most Ranges4::kMax of them).
static bool to_ranges4(const gpt2_model* m, const int64_t* ranges, int n, k::Ranges4* out) {
  if (n < 1 || n > k::Ranges4::kMax || !ranges) return false;
  out->n = n;
  for (int r = 0; r < n; ++r) {
    const int64_t b = ranges[2 * r], e = ranges[2 * r + 1];
    if (b < 0 || e < b || e > m->lay.P || (b % 64) || (e % 64)) return false;
    out->begin[r] = b / 4;
    out->end[r] = e / 4;
  }
  return true;
}

// The update half of the step over the given ranges, with the norm finalised from
// `sumsq` (one device double: the sum of squares of the accumulated gradients).
static int clip_adamw_impl(gpt2_model* m, int32_t step, const k::Ranges4& rg, const double* sumsq, int nparts,
                           bool clear_all_grads, float* grad_norm_out) {
  cudaStream_t s = m->stream;
  const Layout& y = m->lay;
  const size_t pr = prof_begin(m);
  launch_pdl(k::norm_finalize_kernel, dim3(1), dim3(256), 0, s, sumsq, nparts, m->sc(), m->n_micro, y.d.N,
             m->cfg.grad_clip, m->err());
  const double lr = lr_at(m->cfg, step);
  const double t = (double)step + 1.0;
  const float bc1 = (float)(1.0 - pow((double)m->cfg.beta1, t));
  const float bc2 = (float)(1.0 - pow((double)m->cfg.beta2, t));
  long n4 = 0;
  for (int r = 0; r < rg.n; ++r) n4 += rg.end[r] - rg.begin[r];
  launch_pdl(k::adamw_kernel, dim3(launch::grid_for(n4, 256)), dim3(256), 0, s, m->params(), m->grads(),
             m->at<float>(y.adam_m), m->at<float>(y.adam_v), m->pbf(), rg, y.P1 / 4, m->sc(), (float)lr, m->cfg.beta1,
             m->cfg.beta2, m->cfg.eps, m->cfg.weight_decay, bc1, bc2);
  int nl = 2;
  if (clear_all_grads) {
    if (cudaMemsetAsync(m->grads(), 0, (size_t)y.P * 4, s) != cudaSuccess) return GPT2_ERR_CUDA;
    ++nl;
  }
  prof_end(m, pr, PC_OPT, 34.0 * 4.0 * (double)n4, nl);
  if (cudaGetLastError() != cudaSuccess) return GPT2_ERR_CUDA;
  m->n_micro = 0;
  m->stepped = true;
  if (grad_norm_out) {
    const int st = collect_device_error(m);
    if (cudaMemcpy(grad_norm_out, &m->sc()->last_norm, sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
      return GPT2_ERR_CUDA;
    return st;
  }
  return GPT2_OK;
}

int gpt2_clip_adamw(gpt2_model* m, int32_t step, float* grad_norm_out) {
  if (!m || step < 0) return GPT2_ERR_ARG;
  if (m->n_micro == 0) return GPT2_ERR_STATE;
  const Layout& y = m->lay;
  k::Ranges4 all{};
  all.n = 1;
  all.begin[0] = 0;
  all.end[0] = y.P / 4;
  double* part = m->at<double>(y.norm_part);
  const size_t pr = prof_begin(m);
  launch_pdl(k::sumsq_partial_kernel, dim3(kNormBlocks), dim3(512), 0, m->stream, m->grads(), all, part);
  prof_end(m, pr, PC_OPT, 4.0 * (double)y.P, 1);
  return clip_adamw_impl(m, step, all, part, kNormBlocks, false, grad_norm_out);
}

int gpt2_num_buckets(const gpt2_model* m) { return m ? (int)m->lay.bucket_end.size() : -1; }

int gpt2_bucket_range(const gpt2_model* m, int b, int64_t* begin, int64_t* end) {
  if (!m || !begin || !end) return GPT2_ERR_ARG;
  const Layout& y = m->lay;
  if (b == -1) {
    *begin = 0;
    *end = y.P1;
    return GPT2_OK;
  }
  if (b < 0 || b >= (int)y.bucket_end.size()) return GPT2_ERR_ARG;
  *begin = b == 0 ? y.P1 : y.bucket_end[b - 1];
  *end = y.bucket_end[b];
  return GPT2_OK;
}

int gpt2_set_bucket_events(gpt2_model* m, void* const* events, int n) {
  if (!m) return GPT2_ERR_ARG;
  if (n == 0) {
    m->bucket_events.clear();
    return GPT2_OK;
  }
  if (!events || n != (int)m->lay.bucket_end.size()) return GPT2_ERR_ARG;
  m->bucket_events.assign(n, nullptr);
  for (int i = 0; i < n; ++i) {
    if (!events[i]) { m->bucket_events.clear(); return GPT2_ERR_ARG; }
    m->bucket_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  return GPT2_OK;
}

int gpt2_grad_sumsq(gpt2_model* m, const int64_t* ranges, int n_ranges, double* dev_out) {
  if (!m || !dev_out) return GPT2_ERR_ARG;
  k::Ranges4 rg{};
  if (!to_ranges4(m, ranges, n_ranges, &rg)) return GPT2_ERR_ARG;
  double* part = m->at<double>(m->lay.norm_part);
  long n4 = 0;
  for (int r = 0; r < rg.n; ++r) n4 += rg.end[r] - rg.begin[r];
  const size_t pr = prof_begin(m);
  launch_pdl(k::sumsq_partial_kernel, dim3(kNormBlocks), dim3(512), 0, m->stream, m->grads(), rg, part);
  launch_pdl(k::sum_partials_kernel, dim3(1), dim3(256), 0, m->stream, part, kNormBlocks, dev_out);
  prof_end(m, pr, PC_OPT, 16.0 * (double)n4, 2);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

int gpt2_clip_adamw_ranges(gpt2_model* m, int32_t step, const int64_t* ranges, int n_ranges, const double* dev_sumsq,
                           float* grad_norm_out) {
  if (!m || step < 0 || !dev_sumsq) return GPT2_ERR_ARG;
  if (m->n_micro == 0) return GPT2_ERR_STATE;
  k::Ranges4 rg{};
  if (!to_ranges4(m, ranges, n_ranges, &rg)) return GPT2_ERR_ARG;
  return clip_adamw_impl(m, step, rg, dev_sumsq, 1, true, grad_norm_out);
}

int gpt2_last_step_stats(gpt2_model* m, float* mean_loss_out, float* grad_norm_out) {
  if (!m) return GPT2_ERR_ARG;
  if (!m->stepped) return GPT2_ERR_STATE;
  const int st = collect_device_error(m);
  k::StepScalars h;
  if (cudaMemcpy(&h, m->sc(), sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  if (mean_loss_out) *mean_loss_out = h.last_loss;
  if (grad_norm_out) *grad_norm_out = h.last_norm;
  return st;
}

int gpt2_eval_loss(gpt2_model* m, const int32_t* tokens, const int32_t* targets, int32_t batch, float* loss_out) {
  if (!m || !tokens || !targets || batch <= 0 || !loss_out) return GPT2_ERR_ARG;
  const Dims& d = m->lay.d;
  double* acc = m->at<double>(m->lay.eval_acc);
  if (cudaMemsetAsync(acc, 0, sizeof(double), m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  for (int b0 = 0; b0 < batch; b0 += d.B) {
    const int b = std::min(d.B, batch - b0);
    GPT2_TRY(forward(m, tokens + (size_t)b0 * d.T, targets + (size_t)b0 * d.T, b, false, acc));
  }
  const int st = collect_device_error(m);
  double h = 0.0;
  if (cudaMemcpy(&h, acc, sizeof(double), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  *loss_out = (float)(h / ((double)batch * d.T));
  return st;
}

int gpt2_train_step_host(gpt2_model* m, const int32_t* tokens_host, const int32_t* targets_host, int32_t n_micro,
                         int32_t step, float* mean_loss_out, float* grad_norm_out) {
  if (!m || !tokens_host || !targets_host || n_micro <= 0) return GPT2_ERR_ARG;
  const Dims& d = m->lay.d;
  int32_t* tok = m->at<int32_t>(m->lay.tok);
  int32_t* tgt = m->at<int32_t>(m->lay.tgt);
  const size_t bytes = (size_t)d.N * 4;
  for (int i = 0; i < n_micro; ++i) {
    if (cudaMemcpyAsync(tok, tokens_host + (size_t)i * d.N, bytes, cudaMemcpyHostToDevice, m->stream) != cudaSuccess ||
        cudaMemcpyAsync(tgt, targets_host + (size_t)i * d.N, bytes, cudaMemcpyHostToDevice, m->stream) != cudaSuccess)
      return GPT2_ERR_CUDA;
    GPT2_TRY(gpt2_fwd_bwd(m, tok, tgt, nullptr));
  }
  GPT2_TRY(gpt2_clip_adamw(m, step, nullptr));
  return gpt2_last_step_stats(m, mean_loss_out, grad_norm_out);
}

int gpt2_token_losses(gpt2_model* m, float* host_dst, int64_t n) {
  if (!m || !host_dst || n != m->lay.d.N) return GPT2_ERR_ARG;
  const int st = collect_device_error(m);
  if (cudaMemcpy(host_dst, m->at<float>(m->lay.losses), (size_t)n * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return GPT2_ERR_CUDA;
  return st;
}

float gpt2_lr(const gpt2_model* m, int32_t step) { return m ? (float)lr_at(m->cfg, step) : 0.f; }

double gpt2_schedule_lr(const gpt2_config* cfg, int32_t step) { return cfg ? lr_at(*cfg, step) : -1.0; }

int64_t gpt2_kernel_launches(const gpt2_model* m) { return m ? m->launches : -1; }

int gpt2_profile_enable(gpt2_model* m, int on) {
  if (!m) return GPT2_ERR_ARG;
  if (cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  Profiler& p = m->prof;
  p.on = on != 0;
  p.used = 0;
  p.pending.clear();
  for (int i = 0; i < PC_N; ++i) { p.ms[i] = 0; p.work[i] = 0; p.n[i] = 0; }
  return GPT2_OK;
}

int gpt2_profile_num_classes(void) { return PC_N; }

const char* gpt2_profile_class_name(int cls) { return (cls >= 0 && cls < PC_N) ? kProfNames[cls] : ""; }

int gpt2_profile_read(gpt2_model* m, int cls, double* ms, int64_t* launches, double* work) {
  if (!m || cls < 0 || cls >= PC_N) return GPT2_ERR_ARG;
  Profiler& p = m->prof;
  if (!p.pending.empty()) {
    if (cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
    for (const Profiler::Entry& e : p.pending) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, p.ev[e.ev], p.ev[e.ev + 1]) != cudaSuccess) return GPT2_ERR_CUDA;
      p.ms[e.cls] += t;
      p.work[e.cls] += e.work;
      p.n[e.cls] += 1;
    }
    p.pending.clear();
    p.used = 0;
  }
  if (ms) *ms = p.ms[cls];
  if (launches) *launches = p.n[cls];
  if (work) *work = p.work[cls];
  return GPT2_OK;
}

int gpt2_num_tensors(const gpt2_model* m) { return m ? (int)m->tensors.size() : 0; }

int gpt2_tensor_info(const gpt2_model* m, int idx, const char** name, int64_t shape[2], int* ndim) {
  if (!m || idx < 0 || idx >= (int)m->tensors.size()) return GPT2_ERR_ARG;
  const NamedTensor& t = m->tensors[idx];
  if (name) *name = t.name.c_str();
  if (shape) { shape[0] = t.shape[0]; shape[1] = t.shape[1]; }
  if (ndim) *ndim = t.ndim;
  return GPT2_OK;
}

static float* state_array(gpt2_model* m, int what) {
  switch (what) {
    case GPT2_PARAMS: return m->params();
    case GPT2_GRADS: return m->grads();
    case GPT2_ADAM_M: return m->at<float>(m->lay.adam_m);
    case GPT2_ADAM_V: return m->at<float>(m->lay.adam_v);
    default: return nullptr;
  }
}

int gpt2_state_device_ptr(gpt2_model* m, int what, void** dev_ptr, int64_t* count) {
  if (!m || !dev_ptr || !count) return GPT2_ERR_ARG;
  if (what == GPT2_WEIGHTS_BF16) {
    *dev_ptr = m->pbf();
    *count = (int64_t)m->lay.P;
    return GPT2_OK;
  }
  float* base = state_array(m, what);
  if (!base) return GPT2_ERR_ARG;
  *dev_ptr = base;
  *count = (int64_t)m->lay.P;
  return GPT2_OK;
}

int gpt2_read(gpt2_model* m, int what, int idx, float* host_dst) {
  if (!m || !host_dst || idx < 0 || idx >= (int)m->tensors.size()) return GPT2_ERR_ARG;
  float* base = state_array(m, what);
  if (!base) return GPT2_ERR_ARG;
  const NamedTensor& t = m->tensors[idx];
  if (cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  if (cudaMemcpy(host_dst, base + t.off, (size_t)t.n * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  return GPT2_OK;
}

int gpt2_write(gpt2_model* m, int what, int idx, const float* host_src) {
  if (!m || !host_src || idx < 0 || idx >= (int)m->tensors.size()) return GPT2_ERR_ARG;
  float* base = state_array(m, what);
  if (!base) return GPT2_ERR_ARG;
  const NamedTensor& t = m->tensors[idx];
  if (cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  if (cudaMemcpy(base + t.off, host_src, (size_t)t.n * 4, cudaMemcpyHostToDevice) != cudaSuccess) return GPT2_ERR_CUDA;
  if (what == GPT2_PARAMS) {
    launch_pdl(k::to_bf16_kernel, dim3(launch::grid_for(t.n, 256)), dim3(256), 0, m->stream, base + t.off,
               m->pbf() + t.off, t.n);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(m->stream) != cudaSuccess) return GPT2_ERR_CUDA;
  }
  return GPT2_OK;
}

// ---------------------------------------------------------------------------
// op-level entry points (one hot-path step each; see gpt2step_ops.h)
// ---------------------------------------------------------------------------
int gpt2op_linear_fwd(const void* inp, const void* w, const float* bias, const void* resid, void* out, int M, int N,
                      int K, int* dev_err, void* stream) {
  if (!inp || !w || !out || !dev_err) return GPT2_ERR_ARG;
  gemm::Call c = gemm_call(gemm::FWD, resid ? gemm::EPI_RESID : gemm::EPI_STORE, M, N, K, dev_err);
  c.a = static_cast<const bf16*>(inp); c.lda = K; c.b = static_cast<const bf16*>(w); c.ldb = K;
  c.out = static_cast<bf16*>(out); c.ldo = N; c.bias = bias; c.aux = static_cast<const bf16*>(resid); c.ld_aux = N;
  if (resid && !bias) return GPT2_ERR_ARG;
  return gemm2::run(c, static_cast<cudaStream_t>(stream));
}

int gpt2op_linear_fwd_gelu(const void* inp, const void* w, const float* bias, void* pre_out, void* gelu_out, int M,
                           int N, int K, int* dev_err, void* stream) {
  if (!inp || !w || !bias || !pre_out || !gelu_out || !dev_err) return GPT2_ERR_ARG;
  gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_GELU, M, N, K, dev_err);
  c.a = static_cast<const bf16*>(inp); c.lda = K; c.b = static_cast<const bf16*>(w); c.ldb = K;
  c.out = static_cast<bf16*>(pre_out); c.out2 = static_cast<bf16*>(gelu_out); c.ldo = N; c.bias = bias;
  return gemm2::run(c, static_cast<cudaStream_t>(stream));
}

int gpt2op_linear_dgrad(const void* dout, const void* w, const void* gelu_pre, void* din, int M, int N, int K,
                        int* dev_err, void* stream) {
  if (!dout || !w || !din || !dev_err) return GPT2_ERR_ARG;
  // din[M, K] = dout[M, N] . w[N, K]: GEMM with reduction N, output width K
  gemm::Call c = gemm_call(gemm::DGRAD, gelu_pre ? gemm::EPI_DGELU : gemm::EPI_STORE, M, K, N, dev_err);
  c.a = static_cast<const bf16*>(dout); c.lda = N; c.b = static_cast<const bf16*>(w); c.ldb = K;
  c.out = static_cast<bf16*>(din); c.ldo = K; c.aux = static_cast<const bf16*>(gelu_pre); c.ld_aux = K;
  return gemm2::run(c, static_cast<cudaStream_t>(stream));
}

int gpt2op_linear_wgrad(const void* dout, const void* inp, float* dw, int M, int N, int K, int splits, int* dev_err,
                        void* stream) {
  if (!dout || !inp || !dw || !dev_err || splits < 0) return GPT2_ERR_ARG;
  // dw[N, K] += dout[M, N]^T . inp[M, K]: GEMM with reduction M
  gemm::Call c = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, N, K, M, dev_err);
  c.a = static_cast<const bf16*>(dout); c.lda = N; c.b = static_cast<const bf16*>(inp); c.ldb = K;
  c.outf = dw; c.ldf = K; c.force_splits = splits;
  return gemm2::run(c, static_cast<cudaStream_t>(stream));
}

int gpt2op_linear_bwd(const void* dout, const void* w, const void* inp, const void* gelu_pre, void* din, float* dw,
                      float* colsum, int M, int N, int K, int* splits_out, int* dev_err, void* stream) {
  if (!dout || !w || !inp || !din || !dw || !dev_err) return GPT2_ERR_ARG;
  if (M < 256 || M % 64 || N % 256 || K % 256) return GPT2_ERR_ARG;
  if (colsum && !gelu_pre) return GPT2_ERR_ARG;
  // din[M, K] = dout[M, N] . w[N, K]: reduction N, output width K
  gemm::Call cd = gemm_call(gemm::DGRAD, gelu_pre ? gemm::EPI_DGELU : gemm::EPI_STORE, M, K, N, dev_err);
  cd.a = static_cast<const bf16*>(dout); cd.lda = N; cd.b = static_cast<const bf16*>(w); cd.ldb = K;
  cd.out = static_cast<bf16*>(din); cd.ldo = K; cd.aux = static_cast<const bf16*>(gelu_pre); cd.ld_aux = K;
  cd.colsum = colsum;
  // dw[N, K] += dout[M, N]^T . inp[M, K]: reduction M
  gemm::Call cw = gemm_call(gemm::WGRAD, gemm::EPI_ACC_F32, N, K, M, dev_err);
  cw.a = static_cast<const bf16*>(dout); cw.lda = N; cw.b = static_cast<const bf16*>(inp); cw.ldb = K;
  cw.outf = dw; cw.ldf = K;
  if (!gemm2::uses_pair(cd) || !gemm2::uses_pair(cw)) return GPT2_ERR_ARG;
  int nl = 0;
  return gemm2::run_group(cd, cw, static_cast<cudaStream_t>(stream), &nl, splits_out);
}

size_t gpt2op_bias_grad_workspace(int M, int N) { return launch::bias_grad_workspace(M, N); }

int gpt2op_bias_grad(const void* dout, float* db, int M, int N, void* workspace, size_t ws_bytes, void* stream) {
  if (!dout || !db) return GPT2_ERR_ARG;
  return launch::bias_grad(static_cast<const bf16*>(dout), db, M, N, static_cast<float*>(workspace), ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

int gpt2op_layernorm_fwd(const void* x, const float* w, const float* b, void* y, float* mean, float* rstd, int rows,
                         int C, void* stream) {
  if (!x || !w || !b || !y || !mean || !rstd || rows <= 0) return GPT2_ERR_ARG;
  return launch::ln_fwd(static_cast<const bf16*>(x), w, b, static_cast<bf16*>(y), mean, rstd, rows, C,
                        static_cast<cudaStream_t>(stream));
}

size_t gpt2op_layernorm_bwd_workspace(int rows, int C) { return launch::ln_bwd_workspace(rows, C); }

int gpt2op_layernorm_bwd(const void* dy, const void* x, const float* mean, const float* rstd, const float* w,
                         const void* dresid, void* dx, float* dw, float* db, int rows, int C, void* workspace,
                         size_t ws_bytes, void* stream) {
  if (!dy || !x || !mean || !rstd || !w || !dx || !dw || !db || rows <= 0) return GPT2_ERR_ARG;
  return launch::ln_bwd(static_cast<const bf16*>(dy), static_cast<const bf16*>(x), mean, rstd, w,
                        static_cast<const bf16*>(dresid), static_cast<bf16*>(dx), dw, db, nullptr, rows, C,
                        static_cast<float*>(workspace), ws_bytes, static_cast<cudaStream_t>(stream));
}

// LayerNorm backward that allocates nothing and takes no workspace.
//
// Its per-block partial column sums live in one library-wide device array,
// g_ln_bwd_noalloc_scratch, of kLnNoallocScratchFloats floats (2,424,832 bytes).
// Every GPU that loads this library holds that array until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and keeps it; that first call should therefore happen before
// any stream capture. All calls share the array, so calls that overlap on the
// GPU (different streams, or different host threads without ordering) race on
// it. Nothing in it has to start at zero: every launch writes each partial it
// later reads.
namespace noalloc {
constexpr size_t kLnNoallocScratchFloats = (size_t)kLnBwdBlocks * 2 * 1024;
__device__ __align__(256) static float g_ln_bwd_noalloc_scratch[kLnNoallocScratchFloats];
constexpr int kMaxDevices = 64;
static float* g_scratch_addr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up once per device).
static int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPT2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ln_bwd_noalloc_scratch) != cudaSuccess || p == nullptr) return GPT2_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return GPT2_OK;
}
}  // namespace noalloc

size_t gpt2op_layernorm_bwd_noalloc_max_bytes(void) { return noalloc::kLnNoallocScratchFloats * sizeof(float); }

int gpt2op_layernorm_bwd_noalloc(const void* dy, const void* x, const float* mean, const float* rstd, const float* w,
                                 const void* dresid, void* dx, float* dw, float* db, int rows, int C, void* stream) {
  if (!dy || !x || !mean || !rstd || !w || !dx || !dw || !db || rows <= 0) return GPT2_ERR_ARG;
  // the partial sums this launch needs must fit the fixed scratch; refuse before touching the GPU
  if (launch::ln_bwd_workspace(rows, C) > gpt2op_layernorm_bwd_noalloc_max_bytes()) return GPT2_ERR_ARG;
  float* scratch = nullptr;
  const int st = noalloc::scratch_for_current_device(&scratch);
  if (st != GPT2_OK) return st;
  return launch::ln_bwd(static_cast<const bf16*>(dy), static_cast<const bf16*>(x), mean, rstd, w,
                        static_cast<const bf16*>(dresid), static_cast<bf16*>(dx), dw, db, nullptr, rows, C, scratch,
                        gpt2op_layernorm_bwd_noalloc_max_bytes(), static_cast<cudaStream_t>(stream));
}

int gpt2op_attention_fwd(const void* qkv, void* out, float* lse, int B, int T, int H, int hd, int* dev_err,
                         void* stream) {
  if (!qkv || !out || !lse || !dev_err) return GPT2_ERR_ARG;
  return launch::attention_fwd(static_cast<const bf16*>(qkv), static_cast<bf16*>(out), lse, B, T, H, hd, dev_err,
                               static_cast<cudaStream_t>(stream));
}

size_t gpt2op_attention_bwd_workspace(int B, int T, int H, int hd) {
  return (size_t)B * T * H * hd * 4 + (size_t)B * H * T * 32;
}

int gpt2op_attention_bwd(const void* qkv, const void* out, const void* dout, const float* lse, void* dqkv,
                         float* dbias, int B, int T, int H, int hd, void* workspace, size_t ws_bytes, int* dev_err,
                         void* stream) {
  if (!qkv || !out || !dout || !lse || !dqkv || !workspace || !dev_err) return GPT2_ERR_ARG;
  if (ws_bytes < gpt2op_attention_bwd_workspace(B, T, H, hd)) return GPT2_ERR_ARG;
  float* dq_acc = static_cast<float*>(workspace);
  float* Dv = dq_acc + (size_t)B * T * H * hd;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(dq_acc, 0, (size_t)B * T * H * hd * 4, s) != cudaSuccess) return GPT2_ERR_CUDA;
  return launch::attention_bwd(static_cast<const bf16*>(qkv), static_cast<const bf16*>(out),
                               static_cast<const bf16*>(dout), lse, Dv, dq_acc, static_cast<bf16*>(dqkv), dbias, B, T,
                               H, hd, dev_err, s);
}

int gpt2op_softmax_ce(void* logits, const int32_t* targets, float* losses, int N, int V, int Vp, float dscale,
                      int* dev_err, void* stream) {
  if (!logits || !targets || !losses || !dev_err || N <= 0) return GPT2_ERR_ARG;
  return launch::softmax_ce(static_cast<bf16*>(logits), targets, losses, N, V, Vp, dscale, 1, dev_err,
                            static_cast<cudaStream_t>(stream));
}

size_t gpt2op_lm_head_ce_workspace(int N, int Vp) {
  if (N <= 0 || Vp <= 0) return 0;
  return (size_t)N * lse_slots(Vp) * 8;
}

int gpt2op_lm_head_ce(const void* h, const void* wte, const int32_t* targets, void* logits, float* losses, int N,
                      int C, int V, int Vp, float dscale, int write_grad, void* workspace, size_t ws_bytes,
                      int* dev_err, void* stream) {
  if (!h || !wte || !targets || !logits || !losses || !dev_err || N <= 0 || C <= 0 || V <= 0 || V > Vp)
    return GPT2_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_STORE, N, Vp, C, dev_err);
  c.a = static_cast<const bf16*>(h); c.lda = C; c.b = static_cast<const bf16*>(wte); c.ldb = C;
  c.out = static_cast<bf16*>(logits); c.ldo = Vp;
  if (!workspace || ws_bytes < gpt2op_lm_head_ce_workspace(N, Vp) || (reinterpret_cast<uintptr_t>(workspace) & 7) != 0)
    return GPT2_ERR_ARG;
  float2* part = nullptr;
  if (gemm2::uses_pair(c)) {
    part = static_cast<float2*>(workspace);
    c.epi = gemm::EPI_LSE; c.lse_part = part; c.lse_V = V;
  }
  const int st = gemm2::run(c, s);
  if (st != GPT2_OK) return st;
  return launch::softmax_ce(static_cast<bf16*>(logits), targets, losses, N, V, Vp, dscale, write_grad ? 1 : 0,
                            dev_err, s, INT_MIN, part, lse_slots(Vp));
}

int gpt2op_lm_head_loss(const void* h, const void* wte, const int32_t* targets, float* losses, int N, int C, int V,
                        int Vp, void* workspace, size_t ws_bytes, int* dev_err, void* stream) {
  if (!h || !wte || !targets || !losses || !dev_err || N <= 0 || C <= 0 || V <= 0 || V > Vp) return GPT2_ERR_ARG;
  if (!workspace || ws_bytes < gpt2op_lm_head_ce_workspace(N, Vp) || (reinterpret_cast<uintptr_t>(workspace) & 7) != 0)
    return GPT2_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gemm::Call c = gemm_call(gemm::FWD, gemm::EPI_LSE_ONLY, N, Vp, C, dev_err);
  c.a = static_cast<const bf16*>(h); c.lda = C; c.b = static_cast<const bf16*>(wte); c.ldb = C;
  if (!gemm2::uses_pair(c)) return GPT2_ERR_ARG;
  float2* part = static_cast<float2*>(workspace);
  c.lse_part = part; c.lse_V = V; c.lse_tgt = targets; c.lse_tgt_val = losses;
  const int st = gemm2::run(c, s);
  if (st != GPT2_OK) return st;
  return launch::softmax_ce(nullptr, targets, losses, N, V, Vp, 1.0f, 0, dev_err, s, INT_MIN, part, lse_slots(Vp),
                            losses);
}

int gpt2op_softmax_ce_masked(void* logits, const int32_t* targets, float* losses, int N, int V, int Vp,
                             int ignore_index, float dscale, int* dev_err, void* stream) {
  if (!logits || !targets || !losses || !dev_err || N <= 0 || ignore_index == INT_MIN) return GPT2_ERR_ARG;
  return launch::softmax_ce(static_cast<bf16*>(logits), targets, losses, N, V, Vp, dscale, 1, dev_err,
                            static_cast<cudaStream_t>(stream), ignore_index);
}

int gpt2op_wait_selftest(int64_t limit_ns, int* dev_err, void* stream) {
  if (!dev_err || limit_ns < 1000000 || limit_ns > 5000000000LL) return GPT2_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  k::wait_selftest_kernel<<<1, 32, 0, s>>>(dev_err, (unsigned long long)limit_ns);
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) return GPT2_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, dev_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  return status_of_device_word(h);
}

int gpt2op_embedding_fwd(const int32_t* tokens, const void* wte, const void* wpe, void* out, int B, int T, int C, int V,
                         int* dev_err, void* stream) {
  if (!tokens || !wte || !wpe || !out || !dev_err || C % 8) return GPT2_ERR_ARG;
  const long N = (long)B * T;
  launch_pdl(k::embed_fwd_kernel, dim3(launch::grid_for(N * C / 8, 256)), dim3(256), 0,
             static_cast<cudaStream_t>(stream), tokens, static_cast<const bf16*>(wte), static_cast<const bf16*>(wpe),
             static_cast<bf16*>(out), (int)N, T, C, V, dev_err);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

int gpt2op_embedding_bwd(const int32_t* tokens, const void* dx, float* dwte, float* dwpe, int B, int T, int C, int V,
                         void* stream) {
  if (!tokens || !dx || !dwte || !dwpe || C % 8) return GPT2_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long N = (long)B * T;
  launch_pdl(k::embed_bwd_wpe_kernel, dim3((T * C / 8 + 255) / 256), dim3(256), 0, s, static_cast<const bf16*>(dx),
             dwpe, B, T, C);
  launch_pdl(k::embed_bwd_wte_kernel, dim3((int)((N + k::kEmbRows - 1) / k::kEmbRows)), dim3(256), 0, s, tokens,
             static_cast<const bf16*>(dx), dwte, (int)N, C, V);
  return cudaGetLastError() == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

}  // extern "C"
