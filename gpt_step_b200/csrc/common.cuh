// Shared device helpers for the GPT-2 training-step kernels (sm_100a only).
//
// Every wait on an mbarrier is bounded by wall time (%globaltimer): after
// kWaitLimitNs the waiting thread records GPT2_ERR_TIMEOUT in the model's
// device error word and gives up, so a logic error can never hang the GPU.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/gpt2step.h"

typedef __nv_bfloat16 bf16;

#define GPT2_DEV __device__ __forceinline__

// ---------------------------------------------------------------------------
// device error word (bit flags, read and cleared by the host at sync points)
// ---------------------------------------------------------------------------
enum : int {
  DEVERR_TOKEN_RANGE = 1 << 0,
  DEVERR_NONFINITE = 1 << 1,
  DEVERR_TIMEOUT = 1 << 2,
};

static constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

GPT2_DEV unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

GPT2_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

GPT2_DEV uint32_t lane_id() { return threadIdx.x & 31; }

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
GPT2_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

GPT2_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

GPT2_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

GPT2_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

GPT2_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Returns false (and
// records a timeout) if it does not within limit_ns, or as soon as another
// thread of the grid has recorded a timeout.
GPT2_DEV bool mbar_wait_limit(uint32_t bar, uint32_t parity, int* err, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*(volatile int*)err & DEVERR_TIMEOUT) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicOr(err, DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

GPT2_DEV bool mbar_wait(uint32_t bar, uint32_t parity, int* err) {
  return mbar_wait_limit(bar, parity, err, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// TMA (no cluster multicast anywhere in this library)
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------
// A kernel launched by launch_pdl may be scheduled while the kernel before it
// in the stream is still draining. It calls griddep_wait() before its first
// access to global memory that earlier work writes or reads (the wait returns
// once the previous grid has completed and its writes are visible), and
// griddep_trigger() to let the next kernel launch ahead of its own end. In a
// kernel launched without the attribute both are no-ops.
GPT2_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
GPT2_DEV void griddep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Both, at the start of a kernel (after any set-up that touches no global memory).
GPT2_DEV void pdl_begin() {
  griddep_wait();
  griddep_trigger();
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Bring the 128-byte line holding `ptr` (a valid global address) into L2.
GPT2_DEV void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(ptr)));
}
GPT2_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load of box {x..x+bx, y..y+by} into shared memory, completing
// `bytes` of transaction count on `bar`. x is always a multiple of 64 bf16
// elements (128 bytes) at every call site.
GPT2_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)
// ---------------------------------------------------------------------------
GPT2_DEV void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
GPT2_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
GPT2_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
GPT2_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
GPT2_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, one instruction of shape M x N x 16 (bf16).
GPT2_DEV void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread completes.
GPT2_DEV void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// Load 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
GPT2_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Issue a 32-column TMEM load without waiting (pair with tmem_wait_ld()).
GPT2_DEV void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
GPT2_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 2^x with the hardware approximation (MUFU.EX2; flushes denormals).
GPT2_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Paired fp32 arithmetic: sm_100 executes two independent round-to-nearest
// fp32 operations as one instruction (.f32x2); each lane of the result is
// bit-identical to the scalar fmaf / multiply / add.
GPT2_DEV float2 f2_fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
GPT2_DEV float2 f2_mul(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
GPT2_DEV float2 f2_add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// max(a, b, c) in one instruction (sm_100 three-input max).
GPT2_DEV float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Shared-memory matrix descriptor for a tile stored in the canonical
// 128-byte-swizzled layout (TMA SWIZZLE_128B). Strides are in bytes.
GPT2_DEV uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, M x N, per-operand majorness.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// small numeric helpers
// ---------------------------------------------------------------------------
GPT2_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
GPT2_DEV float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// Column sums over a warp's 32 rows: lane l holds row l's 32 values in cs[];
// after a transpose-reduce (31 shuffles) cs[0] of lane l is the sum of column l.
GPT2_DEV void warp_colsum32(float (&cs)[32], int lane) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = upper ? cs[i] : cs[i + k];
      const float keep = upper ? cs[i + k] : cs[i];
      cs[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
}

// Four fp32 atomic adds to 16-byte aligned global memory in one instruction.
GPT2_DEV void red_add_f32x4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

GPT2_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
GPT2_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
GPT2_DEV double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Hardware tanh (MUFU.TANH, max relative error about 2^-11; the GELU results
// are stored in bf16, whose rounding is 2^-9).
GPT2_DEV float tanh_hw(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GPT-2's tanh-approximation GELU and its derivative (fp32 arithmetic).
GPT2_DEV float gelu_f(float u) {
  const float k = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * u * (1.0f + tanh_hw(k * (u + 0.044715f * u * u * u)));
}
// GELU(u) and GELU'(u) from one tanh.
GPT2_DEV void gelu_and_grad_f(float u, float& g, float& d) {
  const float k = 0.7978845608028654f;
  const float t = tanh_hw(k * (u + 0.044715f * u * u * u));
  g = 0.5f * u * (1.0f + t);
  d = 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * k * (1.0f + 3.0f * 0.044715f * u * u);
}
// The same for two values in paired fp32 arithmetic, with the polynomial
// regrouped around s = u^2:
//   w  = u (k + 0.044715 k s)                 (the tanh argument)
//   h  = 0.5 + 0.5 tanh(w),  GELU  = u h
//   GELU' = h + u (0.5 k + 1.5 * 0.044715 k s) (1 - t^2)
GPT2_DEV void gelu_and_grad_f2(float2 u, float2& g, float2& d) {
  const float k = 0.7978845608028654f;
  const float kc = k * 0.044715f;
  const float2 s = f2_mul(u, u);
  const float2 w = f2_mul(u, f2_fma(s, make_float2(kc, kc), make_float2(k, k)));
  const float2 t = make_float2(tanh_hw(w.x), tanh_hw(w.y));
  const float2 h = f2_fma(t, make_float2(0.5f, 0.5f), make_float2(0.5f, 0.5f));
  g = f2_mul(u, h);
  // -(u q) and (t^2 - 1), so that GELU' = h + (-(u q)) (t^2 - 1) is one fused step
  const float2 nuq = f2_mul(u, f2_fma(s, make_float2(-1.5f * kc, -1.5f * kc), make_float2(-0.5f * k, -0.5f * k)));
  const float2 t2m1 = f2_fma(t, t, make_float2(-1.f, -1.f));
  d = f2_fma(nuq, t2m1, h);
}
GPT2_DEV float gelu_grad_f(float u) {
  const float k = 0.7978845608028654f;
  const float t = tanh_hw(k * (u + 0.044715f * u * u * u));
  return 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * k * (1.0f + 3.0f * 0.044715f * u * u);
}

// ---------------------------------------------------------------------------
// host: one-time set-up per device (function attributes are per context)
// ---------------------------------------------------------------------------
// Runs `fn` (returning cudaError_t) once on each device that calls it, with
// that device current; safe to call from several host threads. A failed
// attempt is retried on the next call.
struct PerDeviceOnce {
  static constexpr int kMaxDevices = 64;
  std::atomic<uint64_t> done{0};
  std::mutex mu;
  template <typename Fn>
  cudaError_t run(Fn&& fn) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = fn();
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
  }
};

// Opt `kern` into `bytes` of dynamic shared memory on the current device (once per device).
template <typename K>
inline cudaError_t smem_optin(PerDeviceOnce& once, K* kern, int bytes) {
  return once.run([&] {
    return cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                bytes);
  });
}

// Number of SMs of the current device.
inline int device_sm_count() {
  static std::atomic<int> cached[PerDeviceOnce::kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= PerDeviceOnce::kMaxDevices) return 148;
  int v = cached[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
  cached[dev].store(v, std::memory_order_relaxed);
  return v;
}

// ---------------------------------------------------------------------------
// host: tensor-map encoding through the driver entry point (no libcuda link)
// ---------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
  }();
  return fn;
}

// Row-major 2-D tensor [outer][inner] (row stride ld elements of elem_bytes);
// boxes of box_inner x box_outer elements.
inline bool encode_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
                          uint64_t outer, uint64_t ld, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swz) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((ld * elem_bytes) & 15)) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bulk-group helpers shared by the TMA store / reduce paths.
GPT2_DEV void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
GPT2_DEV void bulk_wait_group_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
template <int N>
GPT2_DEV void bulk_wait_group() { asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory"); }
GPT2_DEV void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Element-wise add of a shared-memory box into global memory (fp32 tensor map).
GPT2_DEV void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
