// Device side of the persistent decode engine (sm_100a).
//
// One CTA per SM, 9 warps: warp 8 is the producer, warps 0-7 are consumers.
//
// Producer.  Walks the CTA's static schedule (every stage of every layer of
// every step) and streams the bytes each tile needs -- packed weight tiles and
// KV-cache chunks -- from HBM into a ring of 32 KB shared-memory slots with
// 1-D bulk copies (cp.async.bulk, completion on an mbarrier).  Weights do not
// depend on activations, so the producer runs ahead of the consumers across
// stage boundaries and keeps HBM busy while the consumers wait on a
// dependency ("Warp / Block Specialization" and "Tile-Level Pipeline" in
// "TileRT speed notes": data-movement warps overlap compute warps so load ->
// barrier -> compute -> barrier is no longer serial).
//
// Consumers.  For each stage: wait for the stage's dependency counter (one
// thread polls with ld.acquire.gpu, bounded in time), stage the activation
// vector into shared memory (with the RMSNorm folded in), then consume the
// ring tiles: GEMV tiles give each warp one row pair over a k-chunk (16-byte
// vector loads from shared memory, fp32 FMA, warp-shuffle reduction at the
// end of the row); attention tiles give each warp 4 positions at a time of a
// flash-decoding chunk with a warp-level online softmax.  Each stage's
// epilogue (RoPE + KV append, SwiGLU, residual add, argmax) runs on the
// reduced values in registers; results go to small L2-resident buffers and
// the stage's counter is released.  Device-side counters therefore replace
// kernel launches as the ordering mechanism ("persistent Engine Kernel";
// "Persistent execution paradigm", section 5.3 on device-side event counters
// replacing grid synchronisation).
//
// Every wait is bounded (globaltimer); on expiry the CTA records
// XLPK_ERR_TIMEOUT, raises the global abort flag, all CTAs leave at their next
// stage boundary, and the producer waits for its bulk copies in flight before
// the CTA exits.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "params.h"
#include "tcgen05.cuh"

namespace xlpk {

// ------------------------------------------------------------------ PTX glue

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
// try_wait with a suspend-time hint: the thread is parked by the hardware
// until the phase completes or about `ns` nanoseconds pass, instead of
// re-issuing the test (which would steal issue slots from the warps that
// share its scheduler).
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Explicit shared-state-space loads.  The stage bodies are separate
// (non-inlined) functions, where the compiler cannot prove that a pointer into
// the ring or the activation buffer addresses shared memory; generic loads
// would take the slower L1TEX path.  Volatile: ring slots are rewritten by
// bulk copies between mbarrier phases.
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds_u2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u1(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a));
  return v;
}
// 2-D tiled TMA load (box of the tensor map at column x, row y) into this
// CTA's shared memory, completing its bytes on `bar`.  x * 2 bytes is a
// multiple of 16 (x is 0 or 64).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
// D += A * B for one 16x8x16 tile: bf16 operands, fp32 accumulate (warp-wide).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
      " {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The same tile with fp16 operands.
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
      " {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
template <bool F16>
__device__ __forceinline__ void mma_16816t(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  if constexpr (F16)
    mma_16816_f16(d, a0, a1, a2, a3, b0, b1);
  else
    mma_16816(d, a0, a1, a2, a3, b0, b1);
}
// Two e4m3 codes (low byte first) -> their exact values as an f16x2 (low half
// first); every e4m3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t r;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(r) : "r"(two_codes));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// Two-term bf16 split of an fp32 pair: x = hi + lo with hi = bf16(x) and
// lo = bf16(x - hi), so hi*k + lo*k carries ~16 significant bits of x into a
// bf16 tensor-core product with an exact bf16 k (K and V entries).
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}
// The same split into fp16 terms (11 significant bits each, for the fp16
// tensor-core operands of FP8 models at batch 8).
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Shared address of element (row r, dim d) of a K or V chunk of P rows as the
// 128-byte-swizzled TMA boxes lay it out: box d/64 holds [P][64 dims]; the
// 16-byte unit u of row r sits at unit u ^ (r % 8).
__device__ __forceinline__ uint32_t sw128_addr(uint32_t base, int P, int r, int d) {
  return base + (d >> 6) * (P * 128) + r * 128 + ((((d & 63) >> 3) ^ (r & 7)) << 4) + ((d & 7) << 1);
}
// Byte (r, c) of an e4m3 K or V chunk: P rows of D bytes as the TMA writes
// them with the 128-byte (D = 128) or 64-byte (D = 64) swizzle, i.e. the
// 16-byte unit c/16 of row r is stored at unit (c/16) ^ (r & 7) or
// (c/16) ^ ((r/2) & 3); the base is 1024-byte aligned.  Either way the eight
// rows a warp quarter reads at one logical unit land in distinct banks.
template <int D>
__device__ __forceinline__ uint32_t kv8_addr(uint32_t base, int r, int c) {
  static_assert(D == 64 || D == 128, "head_dim");
  const int f = D == 128 ? (r & 7) : ((r >> 1) & 3);
  return base + r * D + ((((c >> 4) ^ f) << 4) | (c & 15));
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 1-D bulk copy global -> this CTA's shared memory; completes `bytes` of tx on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void bulk_g2s_nohint(uint32_t dst, const void* src, uint32_t bytes,
                                                uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_volatile(const int* p) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_acquire_sys(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_acquire_s32(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}
// Consumer barrier that also ORs `v` over the consumer threads, so that every
// consumer gets the same answer.  Any decision of the consumers to leave the
// stage loop must be taken this way: the CTA's abort word can be raised at any
// moment (by the producer or by a consumer whose wait gave up), and consumers
// that read it at different moments would otherwise split, some leaving while
// the rest wait forever at the next consumer barrier.
__device__ __forceinline__ bool consumer_sync_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, o;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred o, 1, %2, a;\n\t"
      "selp.u32 %0, 1, 0, o;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kConsumerThreads)
      : "memory");
  return r != 0;
}
// Release all prior writes of this CTA (ordered by a preceding consumer_sync)
// and add `v` to a gpu-scope counter.
__device__ __forceinline__ unsigned release_add(unsigned* p, unsigned v) {
  __threadfence();
  return atomicAdd(p, v);
}

__device__ __forceinline__ int split_point(int c, int n, int G) {
  return static_cast<int>((static_cast<long long>(c) * n) / G);
}
// CTA owning item i when n items are split evenly over G CTAs.
__device__ __forceinline__ int split_owner(int i, int n, int G) {
  return static_cast<int>(((static_cast<long long>(i) + 1) * G - 1) / n);
}

// ------------------------------------------------------------------ shared state

struct alignas(16) SmemCtl {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t act_bar;      // completion of the activation bulk copy
  uint64_t acc_bar;      // batch-8 tensor-core stages: the stage's MMAs have completed
  uint64_t bop_bar;      //   the MMAs of a K window are done with its staged input
  uint64_t fin_bar;      //   every MMA issued has completed (before the columns are freed)
  uint32_t tmem_base;    //   this CTA's tensor-memory columns
  volatile int abort;
  int flag;
  int pad[2];
  float red[kConsumerWarps][kMaxBatch];    // RMSNorm partial sums
  float redv[kConsumerWarps][kMaxBatch];   // LM-head argmax values
  int redi[kConsumerWarps][kMaxBatch];     // LM-head argmax indices
  unsigned long long tacc[8];              // attention trace totals (thread 0)
  // MoE routing of the current layer, computed by this CTA's consumers and
  // read by its producer: route_seq = step * L + layer + 1 once the table is set
  volatile int route_seq;
  int route_exp[kMaxMoeSlots];
  float route_w[kMaxMoeSlots];
  float logits[kMaxExperts];
};
static_assert(sizeof(SmemCtl) <= kMiscSmem, "control block too large");

struct RingPos {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int nslot) {
    if (++slot == nslot) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

struct Ctx {
  uint8_t* ring;
  float* act;
  uint8_t* side;       // epilogue side data (RoPE rows, residual / embedding slices)
  SmemCtl* ctl;
  int c;
  int warp;
  int lane;
  int tid;
  uint32_t act_phase;   // parity of the next activation-copy phase (consumers)
  uint32_t acc_phase;   // batch-8 tensor-core stages: parity of the next acc_bar / bop_bar phase
  uint32_t bop_phase;
};

enum ErrCode : int { kErrNone = 0, kErrBadPage = -1, kErrTimeout = -6, kErrAborted = -7 };

__device__ __forceinline__ void raise_error(const Params& p, int code, int where) {
  if (atomicCAS(p.status, 0, code) == 0) {
    p.status[1] = where;
    p.status[2] = blockIdx.x;
  }
  atomicExch(p.abort_flag, 1);
}

// Value of the control block's route_seq once the MoE routing of (step s,
// layer l) is in its table.
__device__ __forceinline__ int route_want(const Params& p, int s, int l) { return s * p.L + l + 1; }

// Timers of stage internals (trace slots 6..13: the attention stage's phases,
// the other stages' input staging): a diagnostic build's option
// (-DXLPK_TRACE_ATTN); the values they keep live cost the release kernel about
// 2 % of a step on the 8B shape.
#ifdef XLPK_TRACE_ATTN
constexpr bool kTraceAttn = true;
#else
constexpr bool kTraceAttn = false;
#endif

__device__ __forceinline__ int where_code(int kind, int layer, int step) {
  return (step << 16) | ((layer & 0xff) << 8) | (kind & 0xff);
}

// Optional stage trace: stamp k of (step s, stage index si) for this CTA.
__device__ __forceinline__ void trace_stamp(const Params& p, int s, int si, int k) {
  if (p.trace) {
    const size_t n_st = static_cast<size_t>(p.L) * ST_LAYER + 1;
    p.trace[((static_cast<size_t>(s) * n_st + si) * p.G + blockIdx.x) * kTraceSlots + k] = globaltimer();
  }
}
__device__ __forceinline__ int stage_index(const Params& p, int kind, int l) {
  return kind == ST_LM ? p.L * ST_LAYER : l * ST_LAYER + kind;
}

// Bounded wait on a ring barrier phase.  Returns false (and marks the CTA
// aborted) if the global abort flag is raised or the time limit passes.
static __device__ __noinline__ bool ring_wait_slow(const Params& p, SmemCtl* ctl, uint32_t bar,
                                            uint32_t parity, int where, int limit_mult = 1) {
  const uint64_t t0 = globaltimer();
  const long long limit = p.spin_limit_ns * limit_mult;
  for (;;) {
    if (p.wait_hint_ns ? mbar_try_wait_suspend(bar, parity, p.wait_hint_ns) : mbar_try_wait(bar, parity))
      return true;
    if (ctl->abort) return false;
    if (ld_volatile(p.abort_flag)) {
      ctl->abort = 1;
      return false;
    }
    if (static_cast<long long>(globaltimer() - t0) > limit) {
      raise_error(p, kErrTimeout, where);
      ctl->abort = 1;
      return false;
    }
  }
}

// Wait for a bulk copy's barrier phase regardless of the abort state.  Copies
// only read device memory and always complete; the bound (at least 2 s,
// independent of the dependency-wait limit) only guards against a device that
// stopped making progress.
static __device__ __noinline__ void copy_wait(const Params& p, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  const long long limit = p.spin_limit_ns > 2000000000LL ? p.spin_limit_ns : 2000000000LL;
  while (!(p.wait_hint_ns ? mbar_try_wait_suspend(bar, parity, p.wait_hint_ns) : mbar_try_wait(bar, parity))) {
    if (static_cast<long long>(globaltimer() - t0) > limit) break;
  }
}

__device__ __forceinline__ bool ring_wait(const Params& p, SmemCtl* ctl, uint32_t bar,
                                          uint32_t parity, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  return ring_wait_slow(p, ctl, bar, parity, where);
}

// Bounded wait (one thread) until *cnt >= target (wrap-safe).
static __device__ __noinline__ bool counter_wait_slow(const Params& p, SmemCtl* ctl, const unsigned* cnt,
                                               unsigned target, int where) {
  const uint64_t t0 = globaltimer();
  unsigned nap = 16;
  for (unsigned it = 1;; ++it) {
    __nanosleep(nap);               // back off: each poll is an L2 round trip
    if (nap < 128) nap <<= 1;
    if (static_cast<int>(ld_acquire(cnt) - target) >= 0) return true;
    if (ctl->abort) return false;
    if ((it & 15u) == 0) {
      if (ld_volatile(p.abort_flag)) {
        ctl->abort = 1;
        return false;
      }
      if (static_cast<long long>(globaltimer() - t0) > p.spin_limit_ns) {
        raise_error(p, kErrTimeout, where);
        ctl->abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool counter_wait(const Params& p, SmemCtl* ctl, const unsigned* cnt,
                                             unsigned target, int where) {
  if (static_cast<int>(ld_acquire(cnt) - target) >= 0) return true;
  return counter_wait_slow(p, ctl, cnt, target, where);
}

// Consumers: thread 0 waits, everyone learns the outcome.  Returns false if aborted.
__device__ __forceinline__ bool stage_wait(const Params& p, Ctx& cx, const unsigned* cnt,
                                           unsigned target, int where, bool fused) {
  if (cx.tid == 0) {
    const int s = where >> 16, kind = where & 0xff, l = (where >> 8) & 0xff;
    trace_stamp(p, s, stage_index(p, kind, l), 0);
    if (fused && !counter_wait(p, cx.ctl, cnt, target, where)) cx.ctl->abort = 1;
    trace_stamp(p, s, stage_index(p, kind, l), 1);
  }
  return !consumer_sync_any(cx.ctl->abort != 0);
}

// ------------------------------------------------------------------ serve mode

// Whether launch step s of a serve launch may run: 1 (requested), -1 (every
// CTA stops at or before s), 0 (not decided yet).
__device__ __forceinline__ int serve_state(const Params& p, int s) {
  if (static_cast<int>(ld_acquire(p.serve_req_dev) - static_cast<unsigned>(p.serve_step0 + s + 1)) >= 0) return 1;
  const int st = ld_acquire_s32(p.serve_stop_dev);
  return st >= 0 && st <= s ? -1 : 0;
}

// Block (bounded) until launch step s is decided; true if it runs.  CTA 0's
// first consumer thread is the poller: it reads the host-mapped request word,
// forwards it, and decides the stop after serve_idle_ns without a request or
// when the host asks to leave; every other waiter follows the device words,
// with a limit above the poller's.
static __device__ __noinline__ bool serve_gate(const Params& p, SmemCtl* ctl, int s, bool poller) {
  const unsigned want = static_cast<unsigned>(p.serve_step0 + s + 1);
  const uint64_t t0 = globaltimer();
  unsigned nap = 32;
  for (;;) {
    if (poller) {
      const unsigned r = ld_acquire_sys(p.serve_req_host);
      if (static_cast<int>(r - want) >= 0) {
        __threadfence();
        atomicMax(p.serve_req_dev, r);
        return true;
      }
      const long long idle = static_cast<long long>(globaltimer() - t0);
      if (*reinterpret_cast<const volatile int*>(p.serve_exit_host) || idle > p.serve_idle_ns) {
        atomicExch(p.serve_stop_dev, s);
        __threadfence();
        return false;
      }
    } else {
      const int st = serve_state(p, s);
      if (st != 0) return st > 0;
      if (static_cast<long long>(globaltimer() - t0) > p.serve_idle_ns + p.spin_limit_ns) {
        raise_error(p, kErrTimeout, where_code(ST_QKV, 0, s) | (1 << 13));
        ctl->abort = 1;
        return false;
      }
    }
    if (ctl->abort || ld_volatile(p.abort_flag)) {
      ctl->abort = 1;
      return false;
    }
    __nanosleep(nap);
    if (nap < 1024) nap <<= 1;
  }
}

// ------------------------------------------------------------------ math

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float dot8_bf16(const uint4 w, const float4 lo, const float4 hi,
                                           float acc) {
  acc = fmaf(bf16_lo(w.x), lo.x, acc);
  acc = fmaf(bf16_hi(w.x), lo.y, acc);
  acc = fmaf(bf16_lo(w.y), lo.z, acc);
  acc = fmaf(bf16_hi(w.y), lo.w, acc);
  acc = fmaf(bf16_lo(w.z), hi.x, acc);
  acc = fmaf(bf16_hi(w.z), hi.y, acc);
  acc = fmaf(bf16_lo(w.w), hi.z, acc);
  acc = fmaf(bf16_hi(w.w), hi.w, acc);
  return acc;
}

// Two e4m3 codes (low byte first) -> two floats, through the CUDA fp8
// conversion to half precision (every e4m3 value is exact in fp16 and fp32).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Sum over 16 e4m3 codes (one 16-byte vector) times 16 fp32 activations
// x0 = elements 0..3, x1 = 4..7, x2 = 8..11, x3 = 12..15.
__device__ __forceinline__ float dot16_e4m3(const uint4 w, const float4 x0, const float4 x1, const float4 x2,
                                            const float4 x3) {
  float acc = 0.f;
  float2 f;
  f = e4m3x2_to_float2(w.x & 0xffffu);  acc = fmaf(f.x, x0.x, fmaf(f.y, x0.y, acc));
  f = e4m3x2_to_float2(w.x >> 16);      acc = fmaf(f.x, x0.z, fmaf(f.y, x0.w, acc));
  f = e4m3x2_to_float2(w.y & 0xffffu);  acc = fmaf(f.x, x1.x, fmaf(f.y, x1.y, acc));
  f = e4m3x2_to_float2(w.y >> 16);      acc = fmaf(f.x, x1.z, fmaf(f.y, x1.w, acc));
  f = e4m3x2_to_float2(w.z & 0xffffu);  acc = fmaf(f.x, x2.x, fmaf(f.y, x2.y, acc));
  f = e4m3x2_to_float2(w.z >> 16);      acc = fmaf(f.x, x2.z, fmaf(f.y, x2.w, acc));
  f = e4m3x2_to_float2(w.w & 0xffffu);  acc = fmaf(f.x, x3.x, fmaf(f.y, x3.y, acc));
  f = e4m3x2_to_float2(w.w >> 16);      acc = fmaf(f.x, x3.z, fmaf(f.y, x3.w, acc));
  return acc;
}

// Two e2m1 codes (one byte, the low nibble first) -> two floats, through the
// CUDA fp4 conversion to half precision (every e2m1 value is exact).
__device__ __forceinline__ float2 e2m1x2_to_float2(uint32_t byte) {
  const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Sum over 16 e2m1 codes (two 32-bit words, element 2j in the low nibble of
// byte j) times 16 fp32 activations x0 = elements 0..3, .., x3 = 12..15.
__device__ __forceinline__ float dot16_e2m1(uint32_t a, uint32_t b, const float4 x0, const float4 x1,
                                           const float4 x2, const float4 x3) {
  float acc = 0.f;
  float2 f;
  f = e2m1x2_to_float2(a & 0xffu);          acc = fmaf(f.x, x0.x, fmaf(f.y, x0.y, acc));
  f = e2m1x2_to_float2((a >> 8) & 0xffu);   acc = fmaf(f.x, x0.z, fmaf(f.y, x0.w, acc));
  f = e2m1x2_to_float2((a >> 16) & 0xffu);  acc = fmaf(f.x, x1.x, fmaf(f.y, x1.y, acc));
  f = e2m1x2_to_float2(a >> 24);            acc = fmaf(f.x, x1.z, fmaf(f.y, x1.w, acc));
  f = e2m1x2_to_float2(b & 0xffu);          acc = fmaf(f.x, x2.x, fmaf(f.y, x2.y, acc));
  f = e2m1x2_to_float2((b >> 8) & 0xffu);   acc = fmaf(f.x, x2.z, fmaf(f.y, x2.w, acc));
  f = e2m1x2_to_float2((b >> 16) & 0xffu);  acc = fmaf(f.x, x3.x, fmaf(f.y, x3.y, acc));
  f = e2m1x2_to_float2(b >> 24);            acc = fmaf(f.x, x3.z, fmaf(f.y, x3.w, acc));
  return acc;
}

__device__ __forceinline__ uint16_t f2bf(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}
// fp32 -> e4m3 code: round to nearest even, saturated to +-448 (NaN stays NaN).
__device__ __forceinline__ uint8_t f2e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void argmax_merge(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

// ------------------------------------------------------------------ activations

// Activation vectors [B][K] (the residual x, the attention output o, the
// SwiGLU output h) are kept in global memory and in shared memory in the same
// "two-plane" fp32 layout, so a stage's input moves as ONE bulk copy and
// lane-consecutive 16-byte reads of 8-element weight vectors are
// conflict-free:  plane 0 holds float4 [B][K/8] = elements 8v..8v+3,
// plane 1 holds elements 8v+4..8v+7.
__host__ __device__ __forceinline__ size_t plane_index(int b, int k, int B, int K) {
  return ((static_cast<size_t>((k >> 2) & 1) * B + b) * (K >> 3) + (k >> 3)) * 4 + (k & 3);
}

// Input vector sources: the residual (two-plane fp32), the pending tokens'
// embedding rows, a plain two-plane vector without RMSNorm (o, h), or the
// fused-FFN layers' residual accumulator (64-bit fixed point, below).
enum ActSrc : int { SRC_RESID = 0, SRC_EMBED = 1, SRC_PLAIN = 2, SRC_FIXED = 3 };

// The residual of the layers whose FFN runs as one fused stage lives in a
// 64-bit fixed-point accumulator with 32 fractional bits: the split-K partial
// sums of the down projection are added with integer atomics, and integer
// addition does not depend on the order in which the CTAs arrive, so every run
// gives the same bits (float atomics would not).  The range is +-2^31, the
// resolution 2^-32; conversions round to nearest.
__device__ __forceinline__ long long to_fixed(float v) { return __float2ll_rn(v * 4294967296.0f); }
__device__ __forceinline__ float from_fixed(long long q) { return __ll2float_rn(q) * 2.3283064365386963e-10f; }

// What the stage's epilogue reads besides its GEMV sums, staged in the CTA's
// side region by the same bulk-copy phase as the input vector, so that no
// epilogue waits on a global load of its own:
//   SIDE_ROPE   cos/sin of this step's position per sequence (QKV)
//   SIDE_RESID  this CTA's rows of the residual x (O-projection, down): two
//               planes of float4, or for the fused-FFN layers rows of the
//               fixed-point accumulator [B][rows_side] int64
//   SIDE_EMBED  this CTA's rows of the pending tokens' embeddings (layer-0 O-projection)
enum SideKind : int { SIDE_NONE = 0, SIDE_ROPE = 1, SIDE_RESID = 2, SIDE_EMBED = 3 };

// Row range [r0, r1) of this CTA in a stage whose matrix has H logical rows
// (row pairs split evenly; with the batch-8 tensor-core tiles, 8-row units).
template <int B>
__device__ __forceinline__ void resid_rows(const Params& p, int c, int& r0, int& r1) {
  if constexpr (B == kMaxBatch) {
    if (p.tc) {
      r0 = 8 * split_point(c, p.H >> 3, p.G);
      r1 = 8 * split_point(c + 1, p.H >> 3, p.G);
      return;
    }
  }
  r0 = 2 * split_point(c, p.H >> 1, p.G);
  r1 = 2 * split_point(c + 1, p.H >> 1, p.G);
}

// The residual as the next layer's QKV stage and the LM head read it: the
// fixed-point accumulator in the fused-FFN layers, else the two-plane x.
__device__ __forceinline__ const void* resid_src(const Params& p) {
  return p.resid_fixed ? static_cast<const void*>(p.xacc) : static_cast<const void*>(p.x);
}

// Stage the input vector and the epilogue's side data in shared memory.  A
// residual / plain source (two-plane layout in global memory, written by other
// CTAs in an earlier stage), the RMSNorm gains and the side data arrive by
// bulk copies on one barrier phase issued right after the dependency wait; the
// embedding rows of layer 0 (bf16) are converted by the threads meanwhile.
// With `gain`, RMSNorm is split: one pass forms v * gain in place and the sum
// of squares; rn[b] = rsqrt(mean(v^2) + eps) is applied to the GEMV sums
// (W (g v) r = W (r g v)), so the stage needs a single consumer barrier.
// `hidden_dbg` (LM stage, CTA 0) receives the raw residual in natural [B][K] order.
//
// SRC_FIXED (the fused-FFN layers' residual accumulator) arrives by the same
// bulk copy phase into a staging area behind the fp32 input (int64 [B][K] at
// act + B*K*4 bytes); the threads convert it from shared memory, one group of 4
// at a time, scaled by the gains they loaded before the wait.  (Reading it
// straight into registers instead kept so many values live that the whole
// kernel's register allocation spilled.)
template <int B>
__device__ __noinline__ void load_act(const Params& p, Ctx& cx, int K, ActSrc src, const void* gsrc_v,
                                      const float* gain, float* hidden_dbg, int side, int s,
                                      float (&rn)[B], int where) {
  const float* gsrc = static_cast<const float*>(gsrc_v);
  const bool direct = src == SRC_FIXED;
  // diagnostic build (XLPK_TRACE_ATTN): thread 0's progress through the input
  // staging in trace slots 6..9 (copies issued, landed, converted, reduced)
  auto tstamp = [&](int k) {
    if (kTraceAttn && p.trace && cx.tid == 0)
      trace_stamp(p, where >> 16, stage_index(p, where & 0xff, (where >> 8) & 0xff), k);
  };
  const int nvK = K >> 3;
  const int n4 = K >> 2;
  float4* act4 = reinterpret_cast<float4*>(cx.act);
  const uint32_t bar = smem_addr(&cx.ctl->act_bar);
  const uint32_t gain_s = smem_addr(cx.act + static_cast<size_t>(B) * K);
  if (cx.tid == 0) {
    // order the other CTAs' global writes (acquired) and this CTA's earlier
    // shared-memory accesses before the async-proxy copies
    asm volatile("fence.proxy.async;" ::: "memory");
    const uint32_t side_s = smem_addr(cx.side);
    int r0 = 0, r1 = 0;
    if (side == SIDE_RESID || side == SIDE_EMBED) resid_rows<B>(p, cx.c, r0, r1);
    int tok[B];
    if (side == SIDE_EMBED)
#pragma unroll
      for (int b = 0; b < B; ++b) tok[b] = __ldcg(p.cur_tok + b);
    // total bytes of this phase
    uint32_t total = 0;
    if (src != SRC_EMBED && !direct) total += static_cast<uint32_t>(B) * K * 4u;
    if (direct) total += static_cast<uint32_t>(B) * K * 8u;
    if (gain && !direct) total += static_cast<uint32_t>(K) * 4u;
    const uint32_t rope_bytes = static_cast<uint32_t>(p.d) * 4u;   // d/2 (cos, sin) pairs
    const int v0 = r0 >> 3, nv = r1 > r0 ? ((r1 - 1) >> 3) - v0 + 1 : 0;
    const int e0 = r0 & ~7, e1 = (r1 + 7) & ~7;
    if (side == SIDE_ROPE) total += B * rope_bytes;
    if (side == SIDE_RESID)
      total += p.resid_fixed ? static_cast<uint32_t>(B) * (r1 - r0) * 8u : static_cast<uint32_t>(B) * 2u * nv * 16u;
    if (side == SIDE_EMBED && r1 > r0) total += static_cast<uint32_t>(B) * (e1 - e0) * 2u;
    tstamp(6);
    mbar_expect_tx(bar, total);
    if (src != SRC_EMBED && !direct)
      bulk_g2s_nohint(smem_addr(cx.act), gsrc, static_cast<uint32_t>(B) * K * 4u, bar);
    if (direct)   // int64 [B][K] staged behind the fp32 area
      bulk_g2s_nohint(smem_addr(cx.act) + static_cast<uint32_t>(B) * K * 4u, gsrc, static_cast<uint32_t>(B) * K * 8u,
                      bar);
    if (gain && !direct) bulk_g2s_nohint(gain_s, gain, static_cast<uint32_t>(K) * 4u, bar);
    if (side == SIDE_ROPE) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        bulk_g2s_nohint(side_s + p.side_rope + b * rope_bytes,
                        p.rope + static_cast<size_t>(p.pos0[b] + s) * (p.d >> 1), rope_bytes, bar);
    } else if (side == SIDE_RESID && p.resid_fixed && r1 > r0) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        bulk_g2s_nohint(side_s + p.side_resid + b * p.rows_side * 8, p.xacc + static_cast<size_t>(b) * p.H + r0,
                        static_cast<uint32_t>(r1 - r0) * 8u, bar);
    } else if (side == SIDE_RESID && nv > 0) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        for (int pl = 0; pl < 2; ++pl)
          bulk_g2s_nohint(side_s + p.side_resid + ((b * 2 + pl) * p.nvr) * 16,
                          p.x + ((static_cast<size_t>(pl) * p.B + b) * (p.H >> 3) + v0) * 4,
                          static_cast<uint32_t>(nv) * 16u, bar);
    } else if (side == SIDE_EMBED && r1 > r0) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        bulk_g2s_nohint(side_s + p.side_embed + b * p.evb,
                        p.embed + static_cast<size_t>(tok[b]) * p.H + e0,
                        static_cast<uint32_t>(e1 - e0) * 2u, bar);
    }
  }
  if constexpr (B <= 2) {   // the fused FFN (and so SRC_FIXED) exists for batch <= 2 only
  if (direct) {
    // the gains of this thread's groups (K <= 4096 in the fused-FFN layers)
    constexpr int GJ = 4;
    float4 g[GJ];
#pragma unroll
    for (int j = 0; j < GJ; ++j) {
      const int q = cx.tid + j * kConsumerThreads;
      g[j] = (gain && q < n4) ? __ldg(reinterpret_cast<const float4*>(gain) + q) : make_float4(1.f, 1.f, 1.f, 1.f);
    }
    if (!cx.ctl->abort) ring_wait(p, cx.ctl, bar, cx.act_phase, where);
    if (cx.ctl->abort) copy_wait(p, bar, cx.act_phase);
    cx.act_phase ^= 1u;
    tstamp(7);
    const uint32_t stage = smem_addr(cx.act) + static_cast<uint32_t>(B) * K * 4u;
    float ss[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      ss[b] = 0.f;
#pragma unroll
      for (int j = 0; j < GJ; ++j) {
        const int q = cx.tid + j * kConsumerThreads;
        if (q < n4) {
          const uint32_t a = stage + static_cast<uint32_t>(b * K + 4 * q) * 8u;
          const uint4 u0 = lds_u4(a), u1 = lds_u4(a + 16);
          const float4 v = make_float4(
              from_fixed(static_cast<long long>((static_cast<unsigned long long>(u0.y) << 32) | u0.x)),
              from_fixed(static_cast<long long>((static_cast<unsigned long long>(u0.w) << 32) | u0.z)),
              from_fixed(static_cast<long long>((static_cast<unsigned long long>(u1.y) << 32) | u1.x)),
              from_fixed(static_cast<long long>((static_cast<unsigned long long>(u1.w) << 32) | u1.z)));
          if (hidden_dbg) *reinterpret_cast<float4*>(hidden_dbg + static_cast<size_t>(b) * K + 4 * q) = v;
          ss[b] = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss[b]))));
          act4[((q & 1) * B + b) * nvK + (q >> 1)] =
              make_float4(v.x * g[j].x, v.y * g[j].y, v.z * g[j].z, v.w * g[j].w);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) rn[b] = 1.f;
    tstamp(8);
    if (gain) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const float t = warp_sum(ss[b]);
        if (cx.lane == 0) cx.ctl->red[cx.warp][b] = t;
      }
      consumer_sync();
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) t += cx.ctl->red[w][b];
        rn[b] = rsqrtf(t / static_cast<float>(K) + p.eps);
      }
    } else {
      consumer_sync();
    }
    tstamp(9);
    return;
  }
  }
  if (src == SRC_EMBED) {
    int tok[B];
#pragma unroll
    for (int b = 0; b < B; ++b) tok[b] = __ldcg(p.cur_tok + b);
    for (int q0 = cx.tid; q0 < n4; q0 += kConsumerThreads * 4) {
      uint2 e[4][B];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int q = q0 + u * kConsumerThreads;
          if (q < n4) e[u][b] = __ldg(reinterpret_cast<const uint2*>(p.embed + static_cast<size_t>(tok[b]) * K) + q);
        }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int q = q0 + u * kConsumerThreads;
          if (q < n4)
            act4[((q & 1) * B + b) * nvK + (q >> 1)] =
                make_float4(bf16_lo(e[u][b].x), bf16_hi(e[u][b].x), bf16_lo(e[u][b].y), bf16_hi(e[u][b].y));
        }
    }
  }
  if (!cx.ctl->abort) ring_wait(p, cx.ctl, bar, cx.act_phase, where);
  // even when aborting, the copies must land before the CTA may exit
  if (cx.ctl->abort) copy_wait(p, bar, cx.act_phase);
  cx.act_phase ^= 1u;
  tstamp(7);
  if (hidden_dbg) {
    if (src == SRC_EMBED) consumer_sync();
    for (int k = cx.tid; k < K; k += kConsumerThreads)
#pragma unroll
      for (int b = 0; b < B; ++b) hidden_dbg[static_cast<size_t>(b) * K + k] = cx.act[plane_index(b, k, B, K)];
    consumer_sync();   // the pass below rewrites the vector in place
  }
#pragma unroll
  for (int b = 0; b < B; ++b) rn[b] = 1.f;
  if (gain) {
    // each thread rewrites exactly the float4s it converted above (same q), so
    // the embedding path needs no barrier before this pass
    float ss[B];
#pragma unroll
    for (int b = 0; b < B; ++b) ss[b] = 0.f;
    for (int q = cx.tid; q < n4; q += kConsumerThreads) {
      const float4 g4 = lds_f4(gain_s + q * 16);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float4& a = act4[((q & 1) * B + b) * nvK + (q >> 1)];
        const float4 x = a;
        ss[b] = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, ss[b]))));
        a = make_float4(x.x * g4.x, x.y * g4.y, x.z * g4.z, x.w * g4.w);
      }
    }
    tstamp(8);
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const float t = warp_sum(ss[b]);
      if (cx.lane == 0) cx.ctl->red[cx.warp][b] = t;
    }
    consumer_sync();
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) t += cx.ctl->red[w][b];
      rn[b] = rsqrtf(t / static_cast<float>(K) + p.eps);
    }
  } else if (src == SRC_EMBED) {
    consumer_sync();
  }
  tstamp(9);
}

// ------------------------------------------------------------------ GEMV stages

// Consumer side: each warp owns one row pair of every tile of a group and
// accumulates it over the group's k-chunks; `epi(pair, acc0, acc1)` runs on
// the reduced sums (identical in every lane).  WF: 0 bf16, 1 e4m3 (fp32 scale
// per 128x128 block), 2 NVFP4 (e4m3 scale per 16 columns, matrix scale per row).
// [q0, q1) overrides the CTA's pair range (default: the even split of m's pairs).
template <int B, int WF, class Epi>
__device__ __noinline__ void consume_gemv_t(const Params& p, Ctx& cx, const Mat& m, RingPos& rp,
                                            int where, const float (&rn)[B], Epi& epi, int q0, int q1) {
  const int NP = m.N >> 1;
  const int p0 = q0 >= 0 ? q0 : split_point(cx.c, NP, p.G);
  const int p1 = q0 >= 0 ? q1 : split_point(cx.c + 1, NP, p.G);
  const int KC = m.KC;
  const int nkc = m.K / KC;
  const int nv = KC >> 3;     // 16-byte vectors per row chunk (bf16)
  const int nvK = m.K >> 3;
  const uint32_t act_lo_s = smem_addr(cx.act);
  const uint32_t act_hi_s = act_lo_s + B * nvK * 16;
  for (int g0 = p0; g0 < p1; g0 += kPairsPerTile) {
    const int gp = min(kPairsPerTile, p1 - g0);
    float a0[B], a1[B];
#pragma unroll
    for (int b = 0; b < B; ++b) a0[b] = a1[b] = 0.f;
    for (int kc = 0; kc < nkc; ++kc) {
      const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
      const bool ok = cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where);
      if constexpr (WF == 2) {
        if (ok && cx.warp < gp) {
          // NVFP4 tile: [2gp rows][KC/2 code bytes] then [2gp rows][KC/16 e4m3
          // scales]; lane vectors of 32 codes (16 bytes) = two 16-column scale
          // blocks, each block's sum scaled once
          const int nv32 = KC >> 5;
          const uint32_t base = smem_addr(cx.ring) + rp.slot * kSlotBytes;
          const uint32_t r0 = base + (2 * cx.warp) * (KC >> 1);
          const uint32_t r1 = r0 + (KC >> 1);
          const uint32_t s0 = base + gp * KC + (2 * cx.warp) * (KC >> 4);
          const uint32_t s1 = s0 + (KC >> 4);
          const uint32_t alo = act_lo_s + ((kc * KC) >> 3) * 16;
          const uint32_t ahi = act_hi_s + ((kc * KC) >> 3) * 16;
#pragma unroll 2
          for (int v = cx.lane; v < nv32; v += 32) {
            const uint4 w0 = lds_u4(r0 + v * 16);
            const uint4 w1 = lds_u4(r1 + v * 16);
            const float2 sc0 = e4m3x2_to_float2(lds_u16(s0 + v * 2));
            const float2 sc1 = e4m3x2_to_float2(lds_u16(s1 + v * 2));
#pragma unroll
            for (int b = 0; b < B; ++b) {
              const uint32_t xv = (b * nvK + 4 * v) * 16;
              const float4 x0 = lds_f4(alo + xv), x1 = lds_f4(ahi + xv);
              const float4 x2 = lds_f4(alo + xv + 16), x3 = lds_f4(ahi + xv + 16);
              const float4 x4 = lds_f4(alo + xv + 32), x5 = lds_f4(ahi + xv + 32);
              const float4 x6 = lds_f4(alo + xv + 48), x7 = lds_f4(ahi + xv + 48);
              a0[b] = fmaf(sc0.x, dot16_e2m1(w0.x, w0.y, x0, x1, x2, x3), a0[b]);
              a0[b] = fmaf(sc0.y, dot16_e2m1(w0.z, w0.w, x4, x5, x6, x7), a0[b]);
              a1[b] = fmaf(sc1.x, dot16_e2m1(w1.x, w1.y, x0, x1, x2, x3), a1[b]);
              a1[b] = fmaf(sc1.y, dot16_e2m1(w1.z, w1.w, x4, x5, x6, x7), a1[b]);
            }
          }
        }
      } else if constexpr (WF == 1) {
        if (ok && cx.warp < gp) {
        // e4m3 tile: lane vectors of 16 codes, each inside one 128-column
        // scale block; the block's sum is scaled once
        const int nv8 = KC >> 4;
        const uint32_t base = smem_addr(cx.ring) + rp.slot * kSlotBytes;
        const uint32_t r0 = base + (2 * cx.warp) * KC;
        const uint32_t r1 = r0 + KC;
        const uint32_t s0 = base + 2 * gp * KC + (2 * cx.warp) * (KC >> 5);
        const uint32_t s1 = s0 + (KC >> 5);
        const uint32_t alo = act_lo_s + ((kc * KC) >> 3) * 16;
        const uint32_t ahi = act_hi_s + ((kc * KC) >> 3) * 16;
#pragma unroll 2
        for (int v = cx.lane; v < nv8; v += 32) {
          const uint4 w0 = lds_u4(r0 + v * 16);
          const uint4 w1 = lds_u4(r1 + v * 16);
          const float sc0 = __uint_as_float(lds_u1(s0 + (v >> 3) * 4));
          const float sc1 = __uint_as_float(lds_u1(s1 + (v >> 3) * 4));
#pragma unroll
          for (int b = 0; b < B; ++b) {
            const float4 x0 = lds_f4(alo + (b * nvK + 2 * v) * 16);
            const float4 x1 = lds_f4(ahi + (b * nvK + 2 * v) * 16);
            const float4 x2 = lds_f4(alo + (b * nvK + 2 * v + 1) * 16);
            const float4 x3 = lds_f4(ahi + (b * nvK + 2 * v + 1) * 16);
            a0[b] = fmaf(sc0, dot16_e4m3(w0, x0, x1, x2, x3), a0[b]);
            a1[b] = fmaf(sc1, dot16_e4m3(w1, x0, x1, x2, x3), a1[b]);
          }
        }
        }
      } else if (ok && cx.warp < gp) {
        const uint32_t r0 = smem_addr(cx.ring) + rp.slot * kSlotBytes + (2 * cx.warp) * nv * 16;
        const uint32_t r1 = r0 + nv * 16;
        const uint32_t alo = act_lo_s + (kc * nv) * 16;
        const uint32_t ahi = act_hi_s + (kc * nv) * 16;
#pragma unroll 4
        for (int v = cx.lane; v < nv; v += 32) {
          const uint4 w0 = lds_u4(r0 + v * 16);
          const uint4 w1 = lds_u4(r1 + v * 16);
#pragma unroll
          for (int b = 0; b < B; ++b) {
            const float4 lo = lds_f4(alo + (b * nvK + v) * 16);
            const float4 hi = lds_f4(ahi + (b * nvK + v) * 16);
            a0[b] = dot8_bf16(w0, lo, hi, a0[b]);
            a1[b] = dot8_bf16(w1, lo, hi, a1[b]);
          }
        }
      }
      __syncwarp();
      // Release the slot only after its copy landed: an aborting consumer
      // stops releasing, so the producer never refills a slot whose copy may
      // still be in flight (it notices the abort at its next wait).
      if (cx.lane == 0 && ok) mbar_arrive(smem_addr(&cx.ctl->empty[rp.slot]));
      rp.next(p.nslot);
    }
    if (cx.warp < gp) {
      // NVFP4: the rows' matrix scales
      const float2 gs = WF == 2 ? __ldg(m.gsc + g0 + cx.warp) : make_float2(1.f, 1.f);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        a0[b] = warp_sum(a0[b]) * (WF == 2 ? rn[b] * gs.x : rn[b]);
        a1[b] = warp_sum(a1[b]) * (WF == 2 ? rn[b] * gs.y : rn[b]);
      }
      epi(g0 + cx.warp, a0, a1, cx.lane);
    }
  }
}

// K-windowed GEMV (the down projection when B x F fp32 inputs would crowd
// out the ring): the CTA's tiles arrive window by window (all its groups'
// chunks of one window, then the next), the activation region holds one window
// of the input at a time (refilled by bulk copy after every consumer has left
// the previous window), and each warp keeps its row pair's sums for every
// group in registers until the last window.  The epilogue's side data (SIDE_RESID)
// comes with the first window.
template <int B, bool FP8, class Epi>
__device__ __noinline__ void consume_gemv_win_t(const Params& p, Ctx& cx, const Mat& m, RingPos& rp, int where,
                                                const float* gsrc, int s, Epi& epi) {
  const int NP = m.N >> 1;
  const int p0 = split_point(cx.c, NP, p.G), p1 = split_point(cx.c + 1, NP, p.G);
  const int np = p1 - p0;
  const int ng = (np + kPairsPerTile - 1) / kPairsPerTile;   // <= kMaxWinGroups (checked at create)
  const int KC = m.KC, nkc = m.K / KC, cw = p.down_win / KC;
  const int nvKfull = m.K >> 3;
  float a0[kMaxWinGroups][B], a1[kMaxWinGroups][B];
#pragma unroll
  for (int gi = 0; gi < kMaxWinGroups; ++gi)
#pragma unroll
    for (int b = 0; b < B; ++b) a0[gi][b] = a1[gi][b] = 0.f;
  const uint32_t bar = smem_addr(&cx.ctl->act_bar);
  for (int w = 0; w * cw < nkc; ++w) {
    const int cww = min(cw, nkc - w * cw);
    const int nvK = (cww * KC) >> 3;   // 8-column vectors of this window
    // every consumer has left the previous window before it is overwritten
    consumer_sync();
    if (cx.tid == 0) {
      asm volatile("fence.proxy.async;" ::: "memory");
      uint32_t total = static_cast<uint32_t>(B) * 2u * nvK * 16u;
      int r0 = 0, r1 = 0, v0 = 0, nv = 0;
      if (w == 0) {
        resid_rows<B>(p, cx.c, r0, r1);
        v0 = r0 >> 3;
        nv = r1 > r0 ? ((r1 - 1) >> 3) - v0 + 1 : 0;
        total += static_cast<uint32_t>(B) * 2u * nv * 16u;
      }
      mbar_expect_tx(bar, total);
      const int wv0 = (w * p.down_win) >> 3;   // first vector of the window in the full input
#pragma unroll
      for (int b = 0; b < B; ++b)
        for (int pl = 0; pl < 2; ++pl)
          bulk_g2s_nohint(smem_addr(cx.act) + ((pl * B + b) * nvK) * 16,
                          gsrc + ((static_cast<size_t>(pl) * B + b) * nvKfull + wv0) * 4,
                          static_cast<uint32_t>(nvK) * 16u, bar);
      if (w == 0 && nv > 0) {
        const uint32_t side_s = smem_addr(cx.side);
#pragma unroll
        for (int b = 0; b < B; ++b)
          for (int pl = 0; pl < 2; ++pl)
            bulk_g2s_nohint(side_s + p.side_resid + ((b * 2 + pl) * p.nvr) * 16,
                            p.x + ((static_cast<size_t>(pl) * p.B + b) * (p.H >> 3) + v0) * 4,
                            static_cast<uint32_t>(nv) * 16u, bar);
      }
    }
    if (!cx.ctl->abort) ring_wait(p, cx.ctl, bar, cx.act_phase, where);
    if (cx.ctl->abort) copy_wait(p, bar, cx.act_phase);
    cx.act_phase ^= 1u;
    const uint32_t act_lo_s = smem_addr(cx.act);
    const uint32_t act_hi_s = act_lo_s + B * nvK * 16;
#pragma unroll
    for (int gi = 0; gi < kMaxWinGroups; ++gi) {
      if (gi >= ng) break;
      const int gp = min(kPairsPerTile, np - gi * kPairsPerTile);
      for (int kc = 0; kc < cww; ++kc) {
        const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
        const bool ok = cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where);
        if constexpr (FP8) {
          if (ok && cx.warp < gp) {
            const int nv8 = KC >> 4;
            const uint32_t base = smem_addr(cx.ring) + rp.slot * kSlotBytes;
            const uint32_t r0 = base + (2 * cx.warp) * KC;
            const uint32_t r1 = r0 + KC;
            const uint32_t s0 = base + 2 * gp * KC + (2 * cx.warp) * (KC >> 5);
            const uint32_t s1 = s0 + (KC >> 5);
            const uint32_t alo = act_lo_s + ((kc * KC) >> 3) * 16;
            const uint32_t ahi = act_hi_s + ((kc * KC) >> 3) * 16;
#pragma unroll 2
            for (int v = cx.lane; v < nv8; v += 32) {
              const uint4 w0 = lds_u4(r0 + v * 16);
              const uint4 w1 = lds_u4(r1 + v * 16);
              const float sc0 = __uint_as_float(lds_u1(s0 + (v >> 3) * 4));
              const float sc1 = __uint_as_float(lds_u1(s1 + (v >> 3) * 4));
#pragma unroll
              for (int b = 0; b < B; ++b) {
                const float4 x0 = lds_f4(alo + (b * nvK + 2 * v) * 16);
                const float4 x1 = lds_f4(ahi + (b * nvK + 2 * v) * 16);
                const float4 x2 = lds_f4(alo + (b * nvK + 2 * v + 1) * 16);
                const float4 x3 = lds_f4(ahi + (b * nvK + 2 * v + 1) * 16);
                a0[gi][b] = fmaf(sc0, dot16_e4m3(w0, x0, x1, x2, x3), a0[gi][b]);
                a1[gi][b] = fmaf(sc1, dot16_e4m3(w1, x0, x1, x2, x3), a1[gi][b]);
              }
            }
          }
        } else if (ok && cx.warp < gp) {
          const int nv = KC >> 3;
          const uint32_t r0 = smem_addr(cx.ring) + rp.slot * kSlotBytes + (2 * cx.warp) * nv * 16;
          const uint32_t r1 = r0 + nv * 16;
          const uint32_t alo = act_lo_s + (kc * nv) * 16;
          const uint32_t ahi = act_hi_s + (kc * nv) * 16;
#pragma unroll 4
          for (int v = cx.lane; v < nv; v += 32) {
            const uint4 w0 = lds_u4(r0 + v * 16);
            const uint4 w1 = lds_u4(r1 + v * 16);
#pragma unroll
            for (int b = 0; b < B; ++b) {
              const float4 lo = lds_f4(alo + (b * nvK + v) * 16);
              const float4 hi = lds_f4(ahi + (b * nvK + v) * 16);
              a0[gi][b] = dot8_bf16(w0, lo, hi, a0[gi][b]);
              a1[gi][b] = dot8_bf16(w1, lo, hi, a1[gi][b]);
            }
          }
        }
        __syncwarp();
        if (cx.lane == 0 && ok) mbar_arrive(smem_addr(&cx.ctl->empty[rp.slot]));
        rp.next(p.nslot);
      }
    }
  }
#pragma unroll
  for (int gi = 0; gi < kMaxWinGroups; ++gi) {
    if (gi >= ng) break;
    const int gp = min(kPairsPerTile, np - gi * kPairsPerTile);
    if (cx.warp < gp) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        a0[gi][b] = warp_sum(a0[gi][b]);
        a1[gi][b] = warp_sum(a1[gi][b]);
      }
      epi(p0 + gi * kPairsPerTile + cx.warp, a0[gi], a1[gi], cx.lane);
    }
  }
}

// ------------------------------------------------------------------ batch-8 tensor-core stages

// The epilogue's side data alone (the batch-8 tensor-core stages stage their
// input themselves): the same bulk copies as load_act's, on the act barrier.
template <int B>
__device__ __noinline__ void load_side(const Params& p, Ctx& cx, int side, int s, int where) {
  if (side == SIDE_NONE) return;
  const uint32_t bar = smem_addr(&cx.ctl->act_bar);
  if (cx.tid == 0) {
    asm volatile("fence.proxy.async;" ::: "memory");
    const uint32_t side_s = smem_addr(cx.side);
    int r0 = 0, r1 = 0;
    resid_rows<B>(p, cx.c, r0, r1);
    const uint32_t rope_bytes = static_cast<uint32_t>(p.d) * 4u;
    const int v0 = r0 >> 3, nv = r1 > r0 ? ((r1 - 1) >> 3) - v0 + 1 : 0;
    const int e0 = r0 & ~7, e1 = (r1 + 7) & ~7;
    uint32_t total = 0;
    if (side == SIDE_ROPE) total = B * rope_bytes;
    if (side == SIDE_RESID) total = static_cast<uint32_t>(B) * 2u * nv * 16u;
    if (side == SIDE_EMBED && r1 > r0) total = static_cast<uint32_t>(B) * (e1 - e0) * 2u;
    mbar_expect_tx(bar, total);
    if (side == SIDE_ROPE) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        bulk_g2s_nohint(side_s + p.side_rope + b * rope_bytes,
                        p.rope + static_cast<size_t>(p.pos0[b] + s) * (p.d >> 1), rope_bytes, bar);
    } else if (side == SIDE_RESID && nv > 0) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        for (int pl = 0; pl < 2; ++pl)
          bulk_g2s_nohint(side_s + p.side_resid + ((b * 2 + pl) * p.nvr) * 16,
                          p.x + ((static_cast<size_t>(pl) * p.B + b) * (p.H >> 3) + v0) * 4,
                          static_cast<uint32_t>(nv) * 16u, bar);
    } else if (side == SIDE_EMBED && r1 > r0) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        bulk_g2s_nohint(side_s + p.side_embed + b * p.evb,
                        p.embed + static_cast<size_t>(__ldcg(p.cur_tok + b)) * p.H + e0,
                        static_cast<uint32_t>(e1 - e0) * 2u, bar);
    }
  }
  if (!cx.ctl->abort) ring_wait(p, cx.ctl, bar, cx.act_phase, where);
  if (cx.ctl->abort) copy_wait(p, bar, cx.act_phase);
  cx.act_phase ^= 1u;
}

// Stage columns [k0, k0 + Kw) of the 8 sequences' input as the MMA's B
// operand: boxes of [16 rows][64 columns] bf16 in the 128-byte-swizzle K-major
// layout, box jb at act + jb * 2048.  Row b (< 8) holds bf16(v) of sequence b
// and row 8 + b the rest, bf16(v - bf16(v)), so one M = 128, N = 16 MMA forms
// both partial products and their sum (accumulator columns b and 8 + b) carries
// about 16 significant bits of each input value instead of 8.  The source is
// the two-plane fp32 layout (or, SRC_EMBED, the pending tokens' bf16 embedding
// rows); with `gain` the values are multiplied by it and each thread's sums of
// squares of the raw values are added to ss (the RMSNorm factor is formed once
// every window has been staged).  `hidden_dbg` receives the raw input.
static __device__ __noinline__ void tc_stage_input(const Params& p, Ctx& cx, ActSrc src, const float* gsrc, int K, int k0,
                                            int Kw, const float* gain, float* hidden_dbg, float (&ss)[kMaxBatch],
                                            bool f16) {
  constexpr int B = kMaxBatch;
  const uint32_t act_s = smem_addr(cx.act);
  const int nv = Kw >> 3;   // 8-column vectors of the window
  int tok[B];
#pragma unroll
  for (int b = 0; b < B; ++b) tok[b] = src == SRC_EMBED ? __ldcg(p.cur_tok + b) : 0;
  // one 8-column vector of all 8 sequences per thread and pass: its 16 (or 8)
  // loads are independent and in flight together
  for (int v = cx.tid; v < nv; v += kConsumerThreads) {
    const int k = k0 + 8 * v;
    float4 lo[B], hi[B];
    if (src == SRC_EMBED) {
      uint4 u[B];
#pragma unroll
      for (int b = 0; b < B; ++b)
        u[b] = __ldg(reinterpret_cast<const uint4*>(p.embed + static_cast<size_t>(tok[b]) * K + k));
#pragma unroll
      for (int b = 0; b < B; ++b) {
        lo[b] = make_float4(bf16_lo(u[b].x), bf16_hi(u[b].x), bf16_lo(u[b].y), bf16_hi(u[b].y));
        hi[b] = make_float4(bf16_lo(u[b].z), bf16_hi(u[b].z), bf16_lo(u[b].w), bf16_hi(u[b].w));
      }
    } else {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        lo[b] = __ldcg(reinterpret_cast<const float4*>(gsrc + plane_index(b, k, B, K)));
        hi[b] = __ldcg(reinterpret_cast<const float4*>(gsrc + plane_index(b, k + 4, B, K)));
      }
    }
    float4 g0 = make_float4(1.f, 1.f, 1.f, 1.f), g1 = g0;
    if (gain) {
      g0 = __ldg(reinterpret_cast<const float4*>(gain + k));
      g1 = __ldg(reinterpret_cast<const float4*>(gain + k + 4));
    }
    const int kk = k - k0, jb = kk >> 6, q = (kk & 63) >> 3;
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const float e[8] = {lo[b].x, lo[b].y, lo[b].z, lo[b].w, hi[b].x, hi[b].y, hi[b].z, hi[b].w};
      if (hidden_dbg)
#pragma unroll
        for (int t = 0; t < 8; ++t) hidden_dbg[static_cast<size_t>(b) * K + k + t] = e[t];
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 8; ++t) acc = fmaf(e[t], e[t], acc);
      ss[b] += acc;
      const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      uint32_t h2[4], l2[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (f16)
          split_f16x2(e[2 * t] * gv[2 * t], e[2 * t + 1] * gv[2 * t + 1], h2[t], l2[t]);
        else
          split_bf16x2(e[2 * t] * gv[2 * t], e[2 * t + 1] * gv[2 * t + 1], h2[t], l2[t]);
      }
      const uint32_t dst = act_s + jb * 2048 + b * 128 + ((q ^ b) << 4);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(h2[0]), "r"(h2[1]), "r"(h2[2]),
                   "r"(h2[3])
                   : "memory");
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 1024), "r"(l2[0]), "r"(l2[1]), "r"(l2[2]),
                   "r"(l2[3])
                   : "memory");
    }
  }
  // the MMAs read the operand through the async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  consumer_sync();
}

// Widen an FP8 tile in its ring slot to fp16 boxes in place: nb e4m3 boxes of
// [rv][128 codes] (+ the rows' scales) become 2*nb fp16 boxes of [rv][64],
// the codes times their block scale rounded to fp16 (11 significant bits;
// the MMAs of FP8 models take fp16 operands), same swizzle.  Every consumer
// thread reads its units before any is overwritten.
static __device__ __noinline__ void tc_widen_fp8(Ctx& cx, uint32_t slot_s, int rv, int nb) {
  constexpr int kMaxUnits = 4;   // 16-byte code units per thread: nb * rv * 8 <= 1024
  const int nu = nb * rv * 8;
  uint4 code[kMaxUnits];
  float sc[kMaxUnits];
#pragma unroll
  for (int t = 0; t < kMaxUnits; ++t) {
    const int i = cx.tid + t * kConsumerThreads;
    if (i < nu) {
      const int j = i / (rv * 8), rem = i - j * rv * 8, r = rem >> 3;
      code[t] = lds_u4(slot_s + i * 16);
      sc[t] = __uint_as_float(lds_u1(slot_s + nb * rv * 128 + (j * rv + r) * 4));
    }
  }
  consumer_sync();
#pragma unroll
  for (int t = 0; t < kMaxUnits; ++t) {
    const int i = cx.tid + t * kConsumerThreads;
    if (i < nu) {
      const int j = i / (rv * 8), rem = i - j * rv * 8, r = rem >> 3, pq = rem & 7;
      const int q = pq ^ (r & 7);                 // logical 16-code unit of the row
      const uint32_t w[4] = {code[t].x, code[t].y, code[t].z, code[t].w};
      uint32_t o[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 a = e4m3x2_to_float2(w[h] & 0xffffu);
        const float2 c = e4m3x2_to_float2(w[h] >> 16);
        o[2 * h] = pack_f16x2(a.x * sc[t], a.y * sc[t]);
        o[2 * h + 1] = pack_f16x2(c.x * sc[t], c.y * sc[t]);
      }
      // columns 16q..16q+15 -> bf16 box 2j + q/4, its 8-column units 2(q%4), 2(q%4)+1
      const uint32_t box = slot_s + (2 * j + (q >> 2)) * rv * 128 + r * 128;
      const int u = 2 * (q & 3);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(box + ((u ^ (r & 7)) << 4)), "r"(o[0]),
                   "r"(o[1]), "r"(o[2]), "r"(o[3])
                   : "memory");
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(box + (((u + 1) ^ (r & 7)) << 4)), "r"(o[4]),
                   "r"(o[5]), "r"(o[6]), "r"(o[7])
                   : "memory");
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  consumer_sync();
}

__device__ __forceinline__ void mbar_arrive_n(uint32_t bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(n) : "memory");
}

// Whether an epilogue is the LM head's (its running argmax is kept per lane in consume_tc).
template <int B> struct EpiLM;
template <class E> struct is_lm_epi { static constexpr bool value = false; };
template <int B> struct is_lm_epi<EpiLM<B>> { static constexpr bool value = true; };

// One batch-8 projection on the tensor cores: the CTA's 8-row units of `m`
// (M-tiles of <= 128 rows, each with kTcAccCols accumulator columns in tensor
// memory: columns b and 8 + b hold sequence b's high and low parts), the input
// staged as the B operand window by window (tc_window: K windows of
// Params::tc_win columns when K is larger, else the whole K), one issuing
// thread (consumer warp 4, lane 0) driving the MMAs and releasing each ring
// slot with tcgen05.commit, then warps 0..3 reading their accumulator rows back
// and running `epi` on each row pair with the RMSNorm factor rn applied.
template <class Epi>
__device__ __noinline__ void consume_tc(const Params& p, Ctx& cx, const Mat& m, RingPos& rp, int where, ActSrc src,
                                        const float* gsrc, const float* gain, float* hidden_dbg, Epi& epi) {
  constexpr int B = kMaxBatch;
  const int fp8 = m.fp8;
  const int U = m.N >> 3;
  const int u0 = split_point(cx.c, U, p.G), u1 = split_point(cx.c + 1, U, p.G);
  const int R = 8 * (u1 - u0), nm = (R + 127) >> 7;
  const int K = m.K, win = tc_window(p.tc_win, K);
  const int bc = tc_box_cols(fp8), kbox = tc_kbox(K, win, fp8);
  const int nw = win > 0 ? (K + win - 1) / win : 1;
  const bool issuer = cx.warp == 4 && cx.lane == 0;
  const uint32_t idesc = tc_idesc(128, kTcAccCols, fp8 != 0);   // FP8 weights: fp16 operands
  const uint32_t tmem = cx.ctl->tmem_base;
  float ss[B];
#pragma unroll
  for (int b = 0; b < B; ++b) ss[b] = 0.f;
  for (int w = 0; w < nw; ++w) {
    const int k0 = w * win, Kw = win > 0 ? min(win, K - k0) : K;
    if (w > 0) {
      // the previous window's MMAs must be done with the staged input
      if (!cx.ctl->abort) ring_wait(p, cx.ctl, smem_addr(&cx.ctl->bop_bar), cx.bop_phase, where);
      cx.bop_phase ^= 1u;
    }
    tc_stage_input(p, cx, src, gsrc, K, k0, Kw, gain, hidden_dbg, ss, fp8 != 0);
    if (issuer) tc_fence_after();
    for (int mt = 0; mt < nm; ++mt) {
      const int rv = min(128, R - 128 * mt);
      const int nb = tc_nb(rv, kbox, fp8);
      const int nt = (Kw / bc) / nb;
      for (int t = 0; t < nt; ++t) {
        const uint32_t slot_s = smem_addr(cx.ring) + rp.slot * kSlotBytes;
        const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
        const uint32_t eb = smem_addr(&cx.ctl->empty[rp.slot]);
        bool ok;
        if (fp8) {
          const bool got = cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where);
          ok = !consumer_sync_any(!got);                 // uniform: the widening is CTA-collective
          if (ok) tc_widen_fp8(cx, slot_s, rv, nb);
        } else {
          ok = issuer ? (cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where)) : true;
        }
        if (issuer && ok) {
          tc_fence_after();
          const int nbx = fp8 ? 2 * nb : nb;            // bf16 boxes of 64 columns in the slot
          const int bx0 = t * nbx;                       // first B-operand box of the tile
#pragma unroll 1
          for (int j = 0; j < nbx; ++j)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc_mma(tmem + mt * kTcAccCols, tc_desc_sw128(slot_s + j * rv * 128 + ks * 32),
                     tc_desc_sw128(smem_addr(cx.act) + (bx0 + j) * 2048 + ks * 32), idesc,
                     (w | t | j | ks) != 0 ? 1u : 0u);
          mbar_arrive_n(eb, kConsumerWarps - 1);
          tc_commit(eb);                                 // the slot is free once these MMAs have read it
        }
        rp.next(p.nslot);
      }
    }
    if (issuer && !cx.ctl->abort) tc_commit(smem_addr(w + 1 < nw ? &cx.ctl->bop_bar : &cx.ctl->acc_bar));
  }
  // the RMSNorm factor over the whole input, while the last MMAs run
  float rn[B];
#pragma unroll
  for (int b = 0; b < B; ++b) rn[b] = 1.f;
  if (gain) {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const float t = warp_sum(ss[b]);
      if (cx.lane == 0) cx.ctl->red[cx.warp][b] = t;
    }
    consumer_sync();
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) t += cx.ctl->red[w][b];
      rn[b] = rsqrtf(t / static_cast<float>(K) + p.eps);
    }
  }
  // accumulators -> epilogue, one row pair at a time
  if (!cx.ctl->abort) ring_wait(p, cx.ctl, smem_addr(&cx.ctl->acc_bar), cx.acc_phase, where);
  cx.acc_phase ^= 1u;
  tc_fence_after();
  const bool aborting = consumer_sync_any(cx.ctl->abort != 0);   // uniform: tcgen05.ld is warp-collective
  if (cx.warp < 4 && !aborting) {
    // The epilogue runs here after all of the stage's MMAs, so nothing hides
    // its latency: every lane works on every pass (lane L: row pair L/8 of a
    // group of four, sequence L%8, values fetched from the pair's rows with
    // one shuffle per sequence), the functor is copied into registers, and the
    // LM head's running argmax is kept per lane and reduced once at the end.
    Epi e = epi;
    constexpr bool kLm = is_lm_epi<Epi>::value;
    const int bl = cx.lane & 7;                        // this lane's sequence
    float rnb = rn[0];
#pragma unroll
    for (int b = 1; b < B; ++b)
      if (b == bl) rnb = rn[b];
    float lm_v = -INFINITY;
    int lm_i = 0x7fffffff;
    for (int mt = 0; mt < nm; ++mt) {
      const int rv = min(128, R - 128 * mt);
      if (cx.warp * 32 >= rv) continue;               // warp-uniform
      uint32_t v[16];
      tc_ld16(tmem + (static_cast<uint32_t>(cx.warp * 32) << 16) + mt * kTcAccCols, v);
      float row[B];   // this lane's accumulator row: high + low part of each sequence
#pragma unroll
      for (int b = 0; b < B; ++b) row[b] = __uint_as_float(v[b]) + __uint_as_float(v[8 + b]);
      const int np = min(16, (rv - cx.warp * 32) >> 1);   // row pairs of this warp's 32 rows
      for (int i0 = 0; i0 < np; i0 += 4) {             // warp-uniform
        const int ip = i0 + (cx.lane >> 3);            // <= 15
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float y0 = __shfl_sync(0xffffffffu, row[b], 2 * ip);
          const float y1 = __shfl_sync(0xffffffffu, row[b], 2 * ip + 1);
          if (b == bl) {
            x0 = y0;
            x1 = y1;
          }
        }
        if (ip >= np) continue;
        x0 *= rnb;
        x1 *= rnb;
        const int pg = 4 * u0 + 64 * mt + 16 * cx.warp + ip;
        if constexpr (kLm) {
          argmax_merge(lm_v, lm_i, x0, 2 * pg);
          argmax_merge(lm_v, lm_i, x1, 2 * pg + 1);
          if (p.logits_out) {
            float* lo = p.logits_out + (static_cast<size_t>(p.logits_overwrite ? 0 : e.s) * p.B + bl) * p.V + 2 * pg;
            lo[0] = x0;
            lo[1] = x1;
          }
        } else {
          // the functor reads element bl of each array on lane bl
          float a0[B], a1[B];
#pragma unroll
          for (int b = 0; b < B; ++b) {
            a0[b] = x0;
            a1[b] = x1;
          }
          e(pg, a0, a1, bl);
        }
      }
    }
    if constexpr (kLm) {
      // lanes bl, bl + 8, bl + 16, bl + 24 hold sequence bl's candidates
#pragma unroll
      for (int o = 8; o < 32; o <<= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, lm_v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, lm_i, o);
        argmax_merge(lm_v, lm_i, v2, i2);
      }
      if (cx.lane < B) argmax_merge(*epi.best_v, *epi.best_i, lm_v, lm_i);
    }
  }
  tc_fence_before();
}

// e4m3 and bf16 tiles are separate instantiations, so neither inner loop
// carries the other's code.
template <int B, bool W4, class Epi>
__device__ __forceinline__ void consume_gemv(const Params& p, Ctx& cx, const Mat& m, RingPos& rp, int where,
                                             const float (&rn)[B], Epi& epi, int q0 = -1, int q1 = -1) {
  if constexpr (W4) {   // NVFP4 kernels (batch 1): every projection's codes and scales
    if (m.fp4) {
      consume_gemv_t<B, 2>(p, cx, m, rp, where, rn, epi, q0, q1);
      return;
    }
  }
  if (m.fp8)
    consume_gemv_t<B, 1>(p, cx, m, rp, where, rn, epi, q0, q1);
  else
    consume_gemv_t<B, 0>(p, cx, m, rp, where, rn, epi, q0, q1);
}

__device__ __forceinline__ size_t kv_row(const Params& p, int l, int b, int g, int t, bool& ok);

// QKV epilogue: RoPE on q/k pairs, q -> workspace, bf16 k/v -> cache at pos.
// The step's cos/sin rows were staged in shared memory (SIDE_ROPE).
template <int B, bool KV8>
struct EpiQKV {
  const Params& p;
  int l, s;
  const float2* rope_s;   // [B][d/2]
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
    const int half = p.d >> 1;
    const int hq = p.nq * half, hk = p.nkv * half;
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lane != b) continue;
      const int pos = p.pos0[b] + s;
      const float r0 = a0[b], r1 = a1[b];
      if (pg < hq + hk) {
        const bool isq = pg < hq;
        const int pp = isq ? pg : pg - hq;
        const int head = pp / half, i = pp - head * half;
        const float2 cs = rope_s[b * half + i];
        const float y0 = r0 * cs.x - r1 * cs.y;
        const float y1 = r0 * cs.y + r1 * cs.x;
        if (isq) {
          float* qd = p.q + (static_cast<size_t>(b) * p.nq + head) * p.d;
          qd[i] = y0;
          qd[i + half] = y1;
        } else {
          bool ok;
          const size_t row = kv_row(p, l, b, head, pos, ok);
          if (KV8 && ok) {
            uint8_t* kd = p.kc8 + row;
            kd[i] = f2e4m3(y0 * p.k_inv);
            kd[i + half] = f2e4m3(y1 * p.k_inv);
          } else if (ok) {
            uint16_t* kd = p.kc + row;
            kd[i] = f2bf(y0);
            kd[i + half] = f2bf(y1);
          } else {
            raise_error(p, kErrBadPage, where_code(ST_QKV, l, s));
          }
        }
      } else {
        const int pv = pg - hq - hk;
        const int head = pv / half, i2 = (pv - head * half) * 2;
        bool ok;
        const size_t row = kv_row(p, l, b, head, pos, ok);
        if (KV8 && ok) {
          const uint16_t packed = static_cast<uint16_t>(f2e4m3(r0 * p.v_inv)) |
                                  static_cast<uint16_t>(static_cast<uint16_t>(f2e4m3(r1 * p.v_inv)) << 8);
          *reinterpret_cast<uint16_t*>(p.vc8 + row + i2) = packed;
        } else if (ok) {
          const uint32_t packed = static_cast<uint32_t>(f2bf(r0)) | (static_cast<uint32_t>(f2bf(r1)) << 16);
          *reinterpret_cast<uint32_t*>(p.vc + row + i2) = packed;
        } else {
          raise_error(p, kErrBadPage, where_code(ST_QKV, l, s));
        }
      }
    }
  }
};

// Residual epilogue: x[b][2pg..2pg+1] += (r0, r1); with `from_embed`, x = E[tok] + r.
// The CTA's rows of x (SIDE_RESID) or of the embedding rows (SIDE_EMBED) were
// staged in shared memory: vectors from v0 of each plane, embedding elements
// from e0.
template <int B>
struct EpiResid {
  const Params& p;
  bool from_embed;
  const uint8_t* side;
  int r0;                  // first row of this CTA's span (its side rows start there)
  float* also = nullptr;   // fused FFN (O-projection): the same sum also to y
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lane != b) continue;
      const int r = 2 * pg;
      float2 base;
      if (from_embed) {
        const uint32_t e =
            *reinterpret_cast<const uint32_t*>(side + p.side_embed + b * p.evb + (r - (r0 & ~7)) * 2);
        base = make_float2(bf16_lo(e), bf16_hi(e));
      } else if (p.resid_fixed) {
        const longlong2 q =
            *reinterpret_cast<const longlong2*>(side + p.side_resid + (b * p.rows_side + (r - r0)) * 8);
        base = make_float2(from_fixed(q.x), from_fixed(q.y));
      } else {
        const float* rs = reinterpret_cast<const float*>(side + p.side_resid);
        base = *reinterpret_cast<const float2*>(rs + ((b * 2 + ((r >> 2) & 1)) * p.nvr + (r >> 3) - (r0 >> 3)) * 4 +
                                                (r & 3));
      }
      const float2 v = make_float2(base.x + a0[b], base.y + a1[b]);
      if (p.resid_fixed)
        *reinterpret_cast<longlong2*>(p.xacc + static_cast<size_t>(b) * p.H + r) = make_longlong2(to_fixed(v.x), to_fixed(v.y));
      else
        *reinterpret_cast<float2*>(p.x + plane_index(b, r, p.B, p.H)) = v;
      if (also) *reinterpret_cast<float2*>(also + plane_index(b, r, p.B, p.H)) = v;
    }
  }
};

// SwiGLU epilogue: h[b][pg] = silu(gate) * up.
template <int B>
struct EpiSwiGLU {
  const Params& p;
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lane != b) continue;
      const float g = a0[b];
      p.h[plane_index(b, pg, p.B, p.F)] = g / (1.f + expf(-g)) * a1[b];
    }
  }
};

// Fused FFN gate/up epilogue: h = silu(gate) * up into this CTA's own slice
// (shared memory, [B][hloc]), pair pg at index pg - p0.
template <int B>
struct EpiSwiGLULocal {
  float* hl;
  int hloc, p0;
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lane != b) continue;
      const float g = a0[b];
      hl[b * hloc + (pg - p0)] = g / (1.f + expf(-g)) * a1[b];
    }
  }
};

// Fused FFN, second half: this CTA's columns [j0, j1) of W_down times its own
// h slice, for all H output rows (split-K over the CTAs), added into the
// residual's fixed-point accumulator with 64-bit integer atomics (the sum does
// not depend on the order of the adds).  Tiles are jt rows of W_down^T (= W_down columns), H
// bf16 each; thread t owns the 8-row vectors t, t + 256, ... of the output.
template <int B>
__device__ __noinline__ void consume_downT(const Params& p, Ctx& cx, RingPos& rp, int where, int j0, int j1,
                                           const float* hl) {
  constexpr int NV = 2;                        // 8-row vectors per thread (H <= 4096)
  const int V8 = p.H >> 3;
  float acc[NV][8][B];
#pragma unroll
  for (int q = 0; q < NV; ++q)
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int b = 0; b < B; ++b) acc[q][e][b] = 0.f;
  const int nj = j1 - j0;
  for (int t0 = 0; t0 < nj; t0 += p.jt) {
    const int ncol = min(p.jt, nj - t0);
    const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
    const bool ok = cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where);
    if (ok) {
      const uint32_t base = smem_addr(cx.ring) + rp.slot * kSlotBytes;
      for (int jj = 0; jj < ncol; ++jj) {
        float hv[B];
#pragma unroll
        for (int b = 0; b < B; ++b) hv[b] = hl[b * p.hloc + t0 + jj];
        const uint32_t col = base + jj * p.H * 2;
#pragma unroll
        for (int q = 0; q < NV; ++q) {
          const int v = cx.tid + q * kConsumerThreads;
          if (v < V8) {
            const uint4 w = lds_u4(col + v * 16);
            const float wf[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                 bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
              for (int b = 0; b < B; ++b) acc[q][e][b] = fmaf(wf[e], hv[b], acc[q][e][b]);
          }
        }
      }
    }
    __syncwarp();
    if (cx.lane == 0 && ok) mbar_arrive(smem_addr(&cx.ctl->empty[rp.slot]));   // this warp is done with it
    rp.next(p.nslot);
  }
  if (!p.resid_fixed) {
    // fp32 residual: vector float atomics (the sum's rounding depends on the
    // order in which the CTAs arrive)
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int v = cx.tid + q * kConsumerThreads;
      if (v < V8) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
          float4* x0 = reinterpret_cast<float4*>(p.x + plane_index(b, 8 * v, p.B, p.H));
          float4* x1 = reinterpret_cast<float4*>(p.x + plane_index(b, 8 * v + 4, p.B, p.H));
          atomicAdd(x0, make_float4(acc[q][0][b], acc[q][1][b], acc[q][2][b], acc[q][3][b]));
          atomicAdd(x1, make_float4(acc[q][4][b], acc[q][5][b], acc[q][6][b], acc[q][7][b]));
        }
      }
    }
    return;
  }
  // The partial sums go to the fixed-point accumulator: first through shared
  // memory (the activation region, unused since the gate/up GEMV), so that
  // each warp's integer adds then cover 32 consecutive rows.
  float* part = cx.act;   // [B][H]
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int v = cx.tid + q * kConsumerThreads;
    if (v < V8) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float4* d = reinterpret_cast<float4*>(part + static_cast<size_t>(b) * p.H + 8 * v);
        d[0] = make_float4(acc[q][0][b], acc[q][1][b], acc[q][2][b], acc[q][3][b]);
        d[1] = make_float4(acc[q][4][b], acc[q][5][b], acc[q][6][b], acc[q][7][b]);
      }
    }
  }
  consumer_sync();
  for (int i = cx.tid; i < B * p.H; i += kConsumerThreads)
    atomicAdd(reinterpret_cast<unsigned long long*>(p.xacc + i), static_cast<unsigned long long>(to_fixed(part[i])));
}

// LM-head epilogue: running (max, lowest index) per sequence in lane b.
template <int B>
struct EpiLM {
  const Params& p;
  int s;
  float* best_v;
  int* best_i;
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lane != b) continue;
      const int row = 2 * pg;
      argmax_merge(*best_v, *best_i, a0[b], row);
      argmax_merge(*best_v, *best_i, a1[b], row + 1);
      if (p.logits_out) {
        float* lo = p.logits_out + (static_cast<size_t>(p.logits_overwrite ? 0 : s) * p.B + b) * p.V + row;
        lo[0] = a0[b];
        lo[1] = a1[b];
      }
    }
  }
};

// MoE router epilogue: the expert logits of this CTA's copy of the router, to
// shared memory (every CTA computes all of them).
template <int B>
struct EpiRouter {
  float* logits;
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
    if (lane == 0) {
      logits[2 * pg] = a0[0];
      logits[2 * pg + 1] = a1[0];
    }
  }
};

// MoE gate/up epilogue over the virtual [slot][pair] space: h = w_slot * silu(gate) * up.
template <int B>
struct EpiMoeGU {
  const Params& p;
  const float* route_w;
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
    if (lane == 0) {
      const float g = a0[0];
      p.h[plane_index(0, pg, 1, p.S * p.Fe)] = route_w[pg / p.Fe] * (g / (1.f + expf(-g)) * a1[0]);
    }
  }
};

// MoE routing of one token (warp 0 of the consumers): softmax over the E
// router logits, the top_k most probable experts (ties -> lower id) with their
// probabilities as weights (not renormalised), shared experts first with
// weight 1.  Writes this CTA's routing table; CTA 0 also records it globally
// (for the kernel-per-op down launch and the caller's experts output).
static __device__ __noinline__ void moe_route(const Params& p, Ctx& cx, int l, int s) {
  constexpr int PER = kMaxExperts / 32;
  float v[PER];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = cx.lane + 32 * i;
    v[i] = e < p.E ? cx.ctl->logits[e] : -INFINITY;
    mx = fmaxf(mx, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    v[i] = (cx.lane + 32 * i < p.E) ? expf(v[i] - mx) : 0.f;
    sum += v[i];
  }
  sum = warp_sum(sum);
#pragma unroll
  for (int i = 0; i < PER; ++i) v[i] = (cx.lane + 32 * i < p.E) ? v[i] / sum : -1.f;
  for (int k = 0; k < p.topk; ++k) {
    float bv = -2.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PER; ++i) argmax_merge(bv, bi, v[i], cx.lane + 32 * i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
      argmax_merge(bv, bi, v2, i2);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (cx.lane + 32 * i == bi) v[i] = -1.f;   // taken
    if (cx.lane == 0) {
      cx.ctl->route_exp[p.nsh + k] = bi;
      cx.ctl->route_w[p.nsh + k] = bv;
      if (cx.c == 0) {
        p.route_exp[l * p.S + p.nsh + k] = bi;
        p.route_w[l * p.S + p.nsh + k] = bv;
        if (p.experts_out) p.experts_out[(static_cast<size_t>(s) * p.L + l) * p.topk + k] = bi;
      }
    }
  }
  if (cx.lane < p.nsh) {
    cx.ctl->route_exp[cx.lane] = p.E + cx.lane;
    cx.ctl->route_w[cx.lane] = 1.f;
    if (cx.c == 0) {
      p.route_exp[l * p.S + cx.lane] = p.E + cx.lane;
      p.route_w[l * p.S + cx.lane] = 1.f;
    }
  }
  __syncwarp();
  if (cx.lane == 0) {
    __threadfence_block();
    cx.ctl->route_seq = route_want(p, s, l);   // the producer may stream the experts now
  }
}

// ------------------------------------------------------------------ attention

// The attention work of one step: items (b, g, chunk j) in that order, chunk j
// covering positions [j*P, (j+1)*P) of sequence b's T = pos0[b] + s + 1.
template <int B>
struct AttnPlan {
  int nch[B];
  int base[B];
  int W;
};

template <int B>
__device__ __forceinline__ void attn_plan(const Params& p, int s, AttnPlan<B>& ap) {
  const int P = p.attn_pos_per_tile;
  int w = 0;
#pragma unroll
  for (int b = 0; b < B; ++b) {
    const int T = p.pos0[b] + s + 1;
    ap.nch[b] = (T + P - 1) / P;
    ap.base[b] = w;
    w += p.nkv * ap.nch[b];
  }
  ap.W = w;
}

// Which CTAs work on which chunks.  With at least one CTA per (sequence, kv
// head), each head gets its own contiguous range of CTAs (head h: CTAs
// [h*G/NH, (h+1)*G/NH)) and its chunks are split evenly over them, so no CTA
// straddles two heads: each CTA loads one q, merges once and arrives once.
// With fewer CTAs than heads the chunks of all heads are split evenly over
// the CTAs in (b, g, j) order, and a CTA may span several heads.
__device__ __forceinline__ bool attn_aligned(const Params& p) { return p.G >= p.B * p.nkv; }

// CTA range [c0, c0 + nc) of head (b, g) in the aligned split.
__device__ __forceinline__ void attn_head_ctas(const Params& p, int b, int g, int& c0, int& nc) {
  const int NH = p.B * p.nkv, h = b * p.nkv + g;
  c0 = split_point(h, p.G, NH);
  nc = split_point(h + 1, p.G, NH) - c0;
}

// Item range [i0, i1) of CTA c (items numbered (b, g, j) in that order).
template <int B>
__device__ __forceinline__ void attn_cta_items(const Params& p, const AttnPlan<B>& ap, int c, int& i0,
                                               int& i1) {
  if (!attn_aligned(p)) {
    i0 = split_point(c, ap.W, p.G);
    i1 = split_point(c + 1, ap.W, p.G);
    return;
  }
  const int NH = p.B * p.nkv;
  const int h = split_owner(c, p.G, NH);   // the head whose CTA range holds c
  const int b = h / p.nkv, g = h - b * p.nkv;
  int c0, nc;
  attn_head_ctas(p, b, g, c0, nc);
  int nch = ap.nch[0], base = ap.base[0];
#pragma unroll
  for (int bb = 1; bb < B; ++bb)
    if (bb == b) {
      nch = ap.nch[bb];
      base = ap.base[bb];
    }
  const int hb = base + g * nch;
  i0 = hb + split_point(c - c0, nch, nc);
  i1 = hb + split_point(c - c0 + 1, nch, nc);
}

template <int B>
__device__ __forceinline__ void attn_item(const Params& p, const AttnPlan<B>& ap, int i, int& b,
                                          int& g, int& j, int& nch, int& base) {
  b = 0;
  nch = ap.nch[0];
  base = ap.base[0];
#pragma unroll
  for (int bb = 1; bb < B; ++bb)
    if (ap.base[bb] <= i) {
      b = bb;
      nch = ap.nch[bb];
      base = ap.base[bb];
    }
  const int r = i - base;
  g = r / nch;
  j = r - g * nch;
}

// Element offset of cache row (layer l, sequence b, kv head g, position t).
// Contiguous cache: [L][B][n_kv][max_seq][d].  Paged cache: a pool
// [L][n_pages][n_kv][P][d] of pages of P positions (P = the attention chunk,
// so a chunk is one page and one TMA box); positions [jP, (j+1)P) of
// sequence b live in pool page page_table[b][j].  A page number outside the
// pool gives offset 0 and ok = false: the caller skips the access and the
// error is reported.
__device__ __forceinline__ size_t kv_row(const Params& p, int l, int b, int g, int t, bool& ok) {
  ok = true;
  if (!p.page_table) return (((static_cast<size_t>(l) * p.B + b) * p.nkv + g) * p.max_seq + t) * p.d;
  const int P = p.attn_pos_per_tile;
  const int j = t / P;
  const int pg = p.page_table[static_cast<size_t>(b) * p.pages_per_seq + j];
  if (static_cast<unsigned>(pg) >= static_cast<unsigned>(p.n_pages)) {
    ok = false;
    return 0;
  }
  return ((((static_cast<size_t>(l) * p.n_pages + pg) * p.nkv + g) * P) + (t - j * P)) * p.d;
}

// Attention scratch in the activation region (the attention stage stages no
// activation vector).  Sizes are in floats.
__host__ __device__ constexpr int attn_scratch_floats(int D, int G) {
  return kConsumerWarps * 16 * kMaxGroup        // p of each warp's positions
         + kConsumerWarps * kMaxGroup * 2       // per-warp (m, l)
         + kConsumerWarps * kMaxGroup * D       // per-warp o
         + 3 * G * kMaxGroup + 2 * kMaxGroup;   // combine: (M, L, weight) per contributor, M*, L*
}


// Flash-decoding over this CTA's chunks of the (sequence, kv head) space on
// warp-level tensor cores.  A chunk is P = 64 (d=128) or 128 (d=64) positions
// whose K and V rows arrive as 128-byte-swizzled TMA boxes.  Warp w takes the
// 16 positions of group pg = w % (P/16) and, for p.V, the dims of half
// ds = w / (P/16) (d=128) or all of them (d=64).  The GQA group's query heads
// fill rows 0..3 of the m16n8k16 A operand, so S = Q K^T for 16 positions is
// 2 n-tiles x d/16 k-steps of mma, the scores stay in the accumulator
// registers for a warp-level online softmax (one row max / sum per head over
// the 16 positions: 2 shuffles each), and P is reused in registers as the A
// operand of O += P V (the accumulator-to-A register reuse of FlashAttention-2).
// The new token's K/V row (written by this step's QKV stage) is patched into
// the chunk in shared memory.
//
// An e4m3 cache (KV8) arrives as two 8 KB boxes of codes (K at the slot's
// start, V 8 KB further).  K codes feed the q.k MMAs straight from shared
// memory: the dot product runs over a permutation of the head dims in which
// k-step ks of lane quad tig covers dims 4*KS*tig + 4*ks + (0..3), so one
// 32-bit word of a K row is the lane's whole B fragment (two f16x2 after an
// exact e4m3 -> f16 conversion), and q is loaded in the same order.  Each warp
// widens the V codes it multiplies (its 16 positions x DW dims) to f16 in the
// bf16 path's swizzled V layout.  The MMAs take fp16 operands: q as two f16
// terms (x 2^8), P as two f16 terms (x 2^12); the scales k_scale and v_scale
// and those powers of two are applied to the scores and to the softmax sum, all
// exact power-of-two multiplies.
template <int B, int D, bool KV8>
__device__ __noinline__ void consume_attn(const Params& p, Ctx& cx, int l, int s, RingPos& rp,
                                         bool fused) {
  static_assert(kMaxGroup == 4, "query heads per kv head fill at most rows 0..3 of the A tile");
  constexpr int P = (kTileBytes / 2) / (D * 2);               // positions per chunk
  constexpr int NPG = P / 16;                                 // position groups per chunk
  constexpr int NDS = kConsumerWarps / NPG;                   // p.V dim splits
  constexpr int DW = D / NDS;                                 // p.V dims per warp
  constexpr int NT = DW / 8;                                  // p.V n-tiles per warp
  constexpr int KS = D / 16;                                  // q.k k-steps
  constexpr int DV = D / 32;                                  // new-row dims per lane
  static_assert(NPG * NDS == kConsumerWarps && NT % 2 == 0, "chunk shape");
  static_assert(!KV8 || (DW == 64 && P * D == 8192), "e4m3 chunk: two 8 KB boxes, 64 dims per warp");
  constexpr float kQMul = 256.f, kPMul = 4096.f;              // e4m3 path: operand pre-scales
  const float smul = KV8 ? p.k_scale * (1.f / kQMul) : 1.f;   // score scale (a power of two)
  const float lmul = KV8 ? kPMul * p.v_inv : 1.f;             // softmax-sum scale (a power of two)
  AttnPlan<B> ap;
  attn_plan<B>(p, s, ap);
  int i0, i1;
  attn_cta_items<B>(p, ap, cx.c, i0, i1);
  const int where = where_code(ST_ATTN, l, s);
  const unsigned S1 = static_cast<unsigned>(p.step_base + s + 1);
  if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_QKV, static_cast<unsigned>(p.G) * S1, where, fused))
    return;
  if (cx.tid == 0) trace_stamp(p, s, stage_index(p, ST_ATTN, l), 2);
  if (i0 >= i1) return;
  const int GQ = p.group;
  const int pg = cx.warp % NPG, ds = cx.warp / NPG;
  const int gid = cx.lane >> 2, tig = cx.lane & 3;
  const int mi = cx.lane >> 3, rr = cx.lane & 7;             // ldmatrix: matrix / row of this lane
  float* sm_ml = cx.act;                                      // [8 warps][4 heads][2]
  float* sm_o = sm_ml + kConsumerWarps * kMaxGroup * 2;       // [8 warps][4 heads][DW]
  const uint32_t ring_s = smem_addr(cx.ring);

  uint32_t qa0[KS], qa2[KS], qb0[KS], qb2[KS];   // q as bf16 hi (a) + lo (b) parts
  float o[NT][4];
  float m_h = -INFINITY, l_h = 0.f;                          // softmax state of head gid
  int seg_b = -1, seg_g = -1, seg_items = 0, seg_nch = 0, seg_base = 0;
  // trace only (thread 0, kept in shared memory to spare registers): ns in
  // ring waits, from the end of the chunks to leaving, q loads, chunk math,
  // merge, arrive, combine; chunks processed
  unsigned long long* ta = cx.ctl->tacc;
  if (kTraceAttn && p.trace && cx.tid == 0)
    for (int k = 0; k < 8; ++k) ta[k] = 0;

  for (int i = i0; i < i1; ++i) {
    int b, g, j, nch, base;
    attn_item<B>(p, ap, i, b, g, j, nch, base);
    if (b != seg_b || g != seg_g) {
      seg_b = b;
      seg_g = g;
      seg_items = 0;
      seg_nch = nch;
      seg_base = base;
      m_h = -INFINITY;
      l_h = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
      const unsigned long long tq0 = (kTraceAttn && p.trace && cx.tid == 0) ? globaltimer() : 0;
      if (KV8 && gid < GQ) {
        // the permuted dim order of the e4m3 K fragments: dims 4*KS*tig + 4*ks + (0..3)
        const float* qs = p.q + (static_cast<size_t>(b) * p.nq + g * GQ + gid) * D + tig * 4 * KS;
        const float sc = p.qk_scale_log2 * kQMul;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const float4 u = __ldcg(reinterpret_cast<const float4*>(qs + ks * 4));
          split_f16x2(u.x * sc, u.y * sc, qa0[ks], qb0[ks]);
          split_f16x2(u.z * sc, u.w * sc, qa2[ks], qb2[ks]);
        }
      } else if (gid < GQ) {
        const float* qs = p.q + (static_cast<size_t>(b) * p.nq + g * GQ + gid) * D;
        const float sc = p.qk_scale_log2;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const float2 u = __ldcg(reinterpret_cast<const float2*>(qs + ks * 16 + tig * 2));
          const float2 v = __ldcg(reinterpret_cast<const float2*>(qs + ks * 16 + 8 + tig * 2));
          split_bf16x2(u.x * sc, u.y * sc, qa0[ks], qb0[ks]);
          split_bf16x2(v.x * sc, v.y * sc, qa2[ks], qb2[ks]);
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) qa0[ks] = qa2[ks] = qb0[ks] = qb2[ks] = 0u;
      }
      if (kTraceAttn && p.trace && cx.tid == 0) ta[2] += globaltimer() - tq0;
    }
    ++seg_items;
    const int T = p.pos0[b] + s + 1;
    const int t_lo = j * P;
    const int npos = min(t_lo + P, T) - t_lo;      // positions of this chunk (incl. the new token)
    const int n_old = min(t_lo + P, T - 1) - t_lo; // positions already in the cache before this step
    const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
    const unsigned long long tw0 = (kTraceAttn && p.trace && cx.tid == 0) ? globaltimer() : 0;
    // warp-uniform: the tile body below is warp-collective (ldmatrix, mma, shuffles)
    const bool have_tile =
        __all_sync(0xffffffffu, cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where));
    if (kTraceAttn && p.trace && cx.tid == 0) {
      ta[0] += globaltimer() - tw0;
    }
    const unsigned long long tc0 = (kTraceAttn && p.trace && cx.tid == 0) ? globaltimer() : 0;
    const uint32_t kt = ring_s + rp.slot * kSlotBytes;
    const uint32_t vt = kt + kTileBytes / 2;
    const uint32_t vt8 = kt + 8192;                 // e4m3 V codes (K codes at kt)
    if (KV8 && have_tile && pg * 16 < npos) {   // warp-uniform
      if (npos > n_old && (n_old >> 4) == pg) {
        // this step's K/V codes of the head into the code chunks
        bool row_ok;
        const size_t row = kv_row(p, l, b, g, T - 1, row_ok);
        constexpr int DB = D / 32;                  // bytes per lane
        if (row_ok) {
          const uint32_t ka = kv8_addr<D>(kt, n_old, cx.lane * DB);
          const uint32_t va = kv8_addr<D>(vt8, n_old, cx.lane * DB);
          if (DB == 4) {
            const unsigned kk = __ldcg(reinterpret_cast<const unsigned*>(p.kc8 + row + cx.lane * DB));
            const unsigned vv = __ldcg(reinterpret_cast<const unsigned*>(p.vc8 + row + cx.lane * DB));
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(ka), "r"(kk) : "memory");
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(va), "r"(vv) : "memory");
          } else {
            const unsigned short kk = __ldcg(reinterpret_cast<const unsigned short*>(p.kc8 + row + cx.lane * DB));
            const unsigned short vv = __ldcg(reinterpret_cast<const unsigned short*>(p.vc8 + row + cx.lane * DB));
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(ka), "h"(kk) : "memory");
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(va), "h"(vv) : "memory");
          }
        }
        __syncwarp();
      }
      // widen this warp's V codes (rows pg*16 + lane%16, 32 dims from ds*DW + 32*(lane/16))
      {
        const int r = pg * 16 + (cx.lane & 15);
        const int c0 = ds * DW + (cx.lane >> 4) * 32;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w0, w1, w2, w3;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                       : "r"(kv8_addr<D>(vt8, r, c0 + 16 * h)));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sw128_addr(vt, P, r, c0 + 16 * h)),
                       "r"(e4m3x2_to_f16x2(w0 & 0xffffu)), "r"(e4m3x2_to_f16x2(w0 >> 16)),
                       "r"(e4m3x2_to_f16x2(w1 & 0xffffu)), "r"(e4m3x2_to_f16x2(w1 >> 16))
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sw128_addr(vt, P, r, c0 + 16 * h + 8)),
                       "r"(e4m3x2_to_f16x2(w2 & 0xffffu)), "r"(e4m3x2_to_f16x2(w2 >> 16)),
                       "r"(e4m3x2_to_f16x2(w3 & 0xffffu)), "r"(e4m3x2_to_f16x2(w3 >> 16))
                       : "memory");
        }
      }
      // the slot is refilled by the async proxy later
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
    }
    if (have_tile && pg * 16 < npos) {   // warp-uniform
      if (!KV8 && npos > n_old && (n_old >> 4) == pg) {
        // this step's K/V entry of the head, from the cache (written by the QKV stage)
        bool row_ok;
        const size_t row = kv_row(p, l, b, g, T - 1, row_ok);   // (a bad page was reported by the producer)
        const uint32_t ka = sw128_addr(kt, P, n_old, cx.lane * DV);
        const uint32_t va = sw128_addr(vt, P, n_old, cx.lane * DV);
        if (!row_ok) {
          // leave the chunk's row as loaded; the decode is abandoned
        } else if (DV == 4) {
          const uint2 kk = __ldcg(reinterpret_cast<const uint2*>(p.kc + row + cx.lane * DV));
          const uint2 vv = __ldcg(reinterpret_cast<const uint2*>(p.vc + row + cx.lane * DV));
          asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(ka), "r"(kk.x), "r"(kk.y) : "memory");
          asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(va), "r"(vv.x), "r"(vv.y) : "memory");
        } else {
          const unsigned kk = __ldcg(reinterpret_cast<const unsigned*>(p.kc + row + cx.lane * DV));
          const unsigned vv = __ldcg(reinterpret_cast<const unsigned*>(p.vc + row + cx.lane * DV));
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(ka), "r"(kk) : "memory");
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(va), "r"(vv) : "memory");
        }
        // the slot is refilled by the async proxy later
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      if (npos < pg * 16 + 16) {
        // Rows past the sequence end hold whatever the cache has there; their
        // softmax weight is 0, but 0 * (inf or NaN) is not, so zero this warp's
        // share of those V rows before they enter P V.
        constexpr int UPR = DW / 8;                       // 16-byte units per row of this warp's dims
        const int r0 = npos;
        for (int u = cx.lane; u < 16 * UPR; u += 32) {
          const int r = pg * 16 + u / UPR;
          if (r >= r0) {
            const uint32_t a = sw128_addr(vt, P, r, ds * DW + (u % UPR) * 8);
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      // ---- S = Q K^T for positions pg*16 .. pg*16+15.  A rows 0..7 carry q's
      // high bf16 terms and rows 8..15 its low terms, so one MMA forms both
      // products: accumulator rows gid and gid + 8 add up to the score.
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KV8) {
        // B fragments straight from the K codes: positions pg*16 + gid (n-tile 0)
        // and pg*16 + 8 + gid (n-tile 1), this quad's 4*KS permuted dims
        uint32_t k0[KS], k1[KS];
#pragma unroll
        for (int h = 0; h < KS / 4; ++h) {
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(k0[4 * h]), "=r"(k0[4 * h + 1]), "=r"(k0[4 * h + 2]), "=r"(k0[4 * h + 3])
                       : "r"(kv8_addr<D>(kt, pg * 16 + gid, tig * 4 * KS + 16 * h)));
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(k1[4 * h]), "=r"(k1[4 * h + 1]), "=r"(k1[4 * h + 2]), "=r"(k1[4 * h + 3])
                       : "r"(kv8_addr<D>(kt, pg * 16 + 8 + gid, tig * 4 * KS + 16 * h)));
        }
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          mma_16816_f16(s0, qa0[ks], qb0[ks], qa2[ks], qb2[ks], e4m3x2_to_f16x2(k0[ks] & 0xffffu),
                        e4m3x2_to_f16x2(k0[ks] >> 16));
          mma_16816_f16(s1, qa0[ks], qb0[ks], qa2[ks], qb2[ks], e4m3x2_to_f16x2(k1[ks] & 0xffffu),
                        e4m3x2_to_f16x2(k1[ks] >> 16));
        }
      } else {
        const int kr = pg * 16 + ((mi >> 1) << 3) + rr;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b00, b01, b10, b11;
          ldsm_x4(sw128_addr(kt, P, kr, ks * 16 + ((mi & 1) << 3)), b00, b01, b10, b11);
          mma_16816(s0, qa0[ks], qb0[ks], qa2[ks], qb2[ks], b00, b01);
          mma_16816(s1, qa0[ks], qb0[ks], qa2[ks], qb2[ks], b10, b11);
        }
      }
      // ---- online softmax of head gid over the 16 positions (4 per lane)
      const int pa = pg * 16 + tig * 2;
      auto score = [&](float hi, float lo) { return KV8 ? (hi + lo) * smul : hi + lo; };
      const float v0 = pa < npos ? score(s0[0], s0[2]) : -INFINITY;
      const float v1 = pa + 1 < npos ? score(s0[1], s0[3]) : -INFINITY;
      const float v2 = pa + 8 < npos ? score(s1[0], s1[2]) : -INFINITY;
      const float v3 = pa + 9 < npos ? score(s1[1], s1[3]) : -INFINITY;
      float mr = fmaxf(fmaxf(v0, v1), fmaxf(v2, v3));
      mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 1));
      mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 2));
      const float mn = fmaxf(m_h, mr);
      const float alpha = (mn == -INFINITY) ? 1.f : exp2f(m_h - mn);
      const float p0 = v0 == -INFINITY ? 0.f : exp2f(v0 - mn);
      const float p1 = v1 == -INFINITY ? 0.f : exp2f(v1 - mn);
      const float p2 = v2 == -INFINITY ? 0.f : exp2f(v2 - mn);
      const float p3 = v3 == -INFINITY ? 0.f : exp2f(v3 - mn);
      float rs = (p0 + p1) + (p2 + p3);
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      l_h = l_h * alpha + (KV8 ? rs * lmul : rs);
      m_h = mn;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        o[nt][0] *= alpha;
        o[nt][1] *= alpha;
        o[nt][2] *= alpha;
        o[nt][3] *= alpha;
      }
      uint32_t pa0, pa2, pb0, pb2;
      if constexpr (KV8) {
        split_f16x2(p0 * kPMul, p1 * kPMul, pa0, pb0);
        split_f16x2(p2 * kPMul, p3 * kPMul, pa2, pb2);
      } else {
        split_bf16x2(p0, p1, pa0, pb0);
        split_bf16x2(p2, p3, pa2, pb2);
      }
      // ---- O += P V for this warp's dims (P's high terms in A rows 0..7, its
      // low terms in rows 8..15: accumulator rows gid + 8 hold the low part)
      const int vr = pg * 16 + ((mi & 1) << 3) + rr;
#pragma unroll
      for (int n2 = 0; n2 < NT / 2; ++n2) {
        uint32_t b00, b01, b10, b11;
        ldsm_x4_t(sw128_addr(vt, P, vr, ds * DW + n2 * 16 + ((mi >> 1) << 3)), b00, b01, b10, b11);
        mma_16816t<KV8>(o[2 * n2], pa0, pb0, pa2, pb2, b00, b01);
        mma_16816t<KV8>(o[2 * n2 + 1], pa0, pb0, pa2, pb2, b10, b11);
      }
    }
    __syncwarp();
    if (kTraceAttn && p.trace && cx.tid == 0) ta[3] += globaltimer() - tc0;
    if (cx.lane == 0 && have_tile) mbar_arrive(smem_addr(&cx.ctl->empty[rp.slot]));
    rp.next(p.nslot);
    // end of a (b, g) segment: merge the 8 warps into this CTA's partial, and
    // let the CTA that completes the head combine every contributor's partial.
    const int ib = seg_base + seg_g * seg_nch;
    const int ie = ib + seg_nch;
    if (i + 1 < i1 && i + 1 < ie) continue;   // the segment goes on
    const unsigned long long tm0 = (kTraceAttn && p.trace && cx.tid == 0) ? globaltimer() : 0;

    // contributors of this head: CTAs c_first .. c_first + ncov - 1 (partial rows 0 .. ncov-1)
    int c_first, ncov;
    if (attn_aligned(p)) {
      attn_head_ctas(p, seg_b, seg_g, c_first, ncov);
    } else {
      c_first = split_owner(ib, ap.W, p.G);
      ncov = split_owner(ie - 1, ap.W, p.G) - c_first + 1;
    }
    const size_t head_row = (static_cast<size_t>(seg_b) * p.nkv + seg_g) * p.G;   // partial rows of this head
    if (tig == 0 && gid < kMaxGroup) {   // lanes 4h hold head h's state
      sm_ml[(cx.warp * kMaxGroup + gid) * 2 + 0] = m_h;
      sm_ml[(cx.warp * kMaxGroup + gid) * 2 + 1] = l_h;
    }
    if (gid < kMaxGroup) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sm_o[(cx.warp * kMaxGroup + gid) * DW + nt * 8 + tig * 2 + 0] = o[nt][0] + o[nt][2];
        sm_o[(cx.warp * kMaxGroup + gid) * DW + nt * 8 + tig * 2 + 1] = o[nt][1] + o[nt][3];
      }
    }
    consumer_sync();
    {
      // merge the position groups: dims of half ds come from warps pg + ds*NPG
      const size_t row = head_row + (cx.c - c_first);
      for (int idx = cx.tid; idx < GQ * D; idx += kConsumerThreads) {
        const int h = idx / D, dd = idx - h * D;
        const int dsd = dd / DW, dl = dd - dsd * DW;
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < NPG; ++q) M = fmaxf(M, sm_ml[((q + dsd * NPG) * kMaxGroup + h) * 2]);
        float Ls = 0.f, Os = 0.f;
#pragma unroll
        for (int q = 0; q < NPG; ++q) {
          const int w = q + dsd * NPG;
          const float mw = sm_ml[(w * kMaxGroup + h) * 2];
          const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
          Ls = fmaf(sm_ml[(w * kMaxGroup + h) * 2 + 1], f, Ls);
          Os = fmaf(sm_o[(w * kMaxGroup + h) * DW + dl], f, Os);
        }
        p.part_o[(row * GQ + h) * D + dd] = Os;
        if (dd == 0) {
          p.part_ml[(row * GQ + h) * 2 + 0] = M;
          p.part_ml[(row * GQ + h) * 2 + 1] = Ls;
        }
      }
      fence_proxy_async_global();   // the combiner may read the partials by bulk copy
    }
    consumer_sync();
    const unsigned long long ta0 = (kTraceAttn && p.trace && cx.tid == 0) ? globaltimer() : 0;
    if (kTraceAttn && p.trace && cx.tid == 0) ta[4] += ta0 - tm0;
    unsigned* arrive = p.cnt + p.cl.attn_arrive + (l * p.B + seg_b) * p.nkv + seg_g;
    if (cx.tid == 0) {
      const unsigned old = release_add(arrive, static_cast<unsigned>(seg_items));
      __threadfence();
      cx.ctl->flag = (old + seg_items == static_cast<unsigned>(seg_nch)) ? 1 : 0;
    }
    consumer_sync();
    const unsigned long long tb0 = (kTraceAttn && p.trace && cx.tid == 0) ? globaltimer() : 0;
    if (kTraceAttn && p.trace && cx.tid == 0) ta[5] += tb0 - ta0;
    if (!cx.ctl->flag) continue;
    // ---- combine: contributors are CTAs c_first .. c_first + ncov - 1 (rows
    // 0..ncov-1); a CTA in that range with no chunk of this head contributes
    // nothing.  Each thread owns 4 consecutive output dims of one query head
    // and reads what it needs straight from L2 with independent loads: all
    // contributors' maxima (one round trip), then their (max, sum) and output
    // vectors (a second round trip); no shared scratch and no barrier.
    // which of the ncov CTAs hold chunks of this head (32-bit arithmetic: the
    // 64-bit division of split_point is far too slow for a per-contributor loop)
    // (each lane decides for contributors lane, lane+32, ...; a ballot shares it)
    uint32_t has_mask[(kMaxCtas + 31) / 32];
#pragma unroll
    for (int w = 0; w < (kMaxCtas + 31) / 32; ++w) {
      const int t = w * 32 + cx.lane;
      bool has = false;
      if (t < ncov) {
        if (attn_aligned(p)) {
          has = seg_nch >= ncov || ((t + 1) * seg_nch) / ncov > (t * seg_nch) / ncov;
        } else {
          const int cc = c_first + t;
          has = max(ib, (cc * ap.W) / p.G) < min(ie, ((cc + 1) * ap.W) / p.G);
        }
      }
      has_mask[w] = __ballot_sync(0xffffffffu, has);
    }
    // The head's partial rows are contiguous in the workspace: when they fit
    // the scratch behind the merge buffers, one bulk copy brings them all in
    // (one round trip); otherwise every thread reads its own from L2.
    float* cp_ml = sm_o + kConsumerWarps * kMaxGroup * DW;     // [ncov][GQ][2]
    float* cp_o = cp_ml + ncov * GQ * 2;                         // [ncov][GQ][D]
    const uint32_t ml_bytes = static_cast<uint32_t>(ncov) * GQ * 2 * 4;
    const uint32_t o_bytes = static_cast<uint32_t>(ncov) * GQ * D * 4;
    // bulk copies need 16-byte aligned addresses and sizes: the (max, sum)
    // block starts at head_row*GQ*8 bytes and is ncov*GQ*8 long
    const bool staged = (cp_o - cx.act) * 4 + o_bytes <= static_cast<uint32_t>(p.act_bytes) &&
                        ((ncov * GQ) & 1) == 0 && ((head_row * GQ) & 1) == 0;
    const float* mlsrc = p.part_ml + head_row * GQ * 2;
    const float* osrc = p.part_o + head_row * GQ * D;
    if (staged) {
      const uint32_t bar = smem_addr(&cx.ctl->act_bar);
      if (cx.tid == 0) {
        asm volatile("fence.proxy.async;" ::: "memory");
        mbar_expect_tx(bar, ml_bytes + o_bytes);
        bulk_g2s_nohint(smem_addr(cp_ml), mlsrc, ml_bytes, bar);
        bulk_g2s_nohint(smem_addr(cp_o), osrc, o_bytes, bar);
      }
      if (!cx.ctl->abort) ring_wait(p, cx.ctl, bar, cx.act_phase, where);
      if (cx.ctl->abort) copy_wait(p, bar, cx.act_phase);
      cx.act_phase ^= 1u;
      mlsrc = cp_ml;
      osrc = cp_o;
    }
    if (kTraceAttn && p.trace && cx.tid == 0) ta[1] += globaltimer() - tb0;
    for (int o4 = cx.tid; o4 < GQ * D / 4; o4 += kConsumerThreads) {
      const int h = (o4 * 4) / D, dd = o4 * 4 - h * D;
      const float* mlh = mlsrc + h * 2;
      const float* oh = osrc + h * D + dd;
      float M = -INFINITY;
      for (int t = 0; t < ncov; ++t) {
        const float mt = staged ? mlh[t * GQ * 2] : __ldcg(mlh + static_cast<size_t>(t) * GQ * 2);
        if ((has_mask[t >> 5] >> (t & 31)) & 1u) M = fmaxf(M, mt);
      }
      float Ls = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int t = 0; t < ncov; ++t) {
        float2 ml;
        float4 ov;
        if (staged) {
          ml = *reinterpret_cast<const float2*>(mlh + t * GQ * 2);
          ov = *reinterpret_cast<const float4*>(oh + t * GQ * D);
        } else {
          ml = __ldcg(reinterpret_cast<const float2*>(mlh + static_cast<size_t>(t) * GQ * 2));
          ov = __ldcg(reinterpret_cast<const float4*>(oh + static_cast<size_t>(t) * GQ * D));
        }
        if (((has_mask[t >> 5] >> (t & 31)) & 1u) && ml.x != -INFINITY) {
          const float w = exp2f(ml.x - M);
          Ls = fmaf(w, ml.y, Ls);
          acc.x = fmaf(w, ov.x, acc.x);
          acc.y = fmaf(w, ov.y, acc.y);
          acc.z = fmaf(w, ov.z, acc.z);
          acc.w = fmaf(w, ov.w, acc.w);
        }
      }
      const float inv = 1.f / Ls;
      *reinterpret_cast<float4*>(p.o + plane_index(seg_b, (seg_g * GQ + h) * D + dd, p.B, p.nq * D)) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (kTraceAttn && p.trace && cx.tid == 0) ta[7] += globaltimer() - tb0;
    fence_proxy_async_global();   // o is read by bulk copies
    consumer_sync();
    if (cx.tid == 0) {
      // reset the arrival count for the next step (ordered before the
      // release below, which the next step's contributors wait behind)
      *reinterpret_cast<volatile unsigned*>(arrive) = 0u;
      release_add(p.cnt + l * ST_LAYER + ST_ATTN, 1u);
      if (kTraceAttn && p.trace) {
        const unsigned long long te = globaltimer();
        ta[6] += te - tb0;
      }
    }
  }
  if (kTraceAttn && p.trace && cx.tid == 0) {
    const size_t n_st = static_cast<size_t>(p.L) * ST_LAYER + 1;
    unsigned long long* e =
        p.trace + ((static_cast<size_t>(s) * n_st + stage_index(p, ST_ATTN, l)) * p.G + blockIdx.x) * kTraceSlots;
    for (int k = 0; k < 8; ++k) e[6 + k] = ta[k];
    for (int k = 0; k < 8; ++k) ta[k] = 0;
  }
}

// ------------------------------------------------------------------ stages

__device__ __forceinline__ const Mat& stage_mat(const LayerParams& L, int kind) {
  return kind == ST_QKV ? L.qkv : kind == ST_OPROJ ? L.o : kind == ST_GATEUP ? L.gu : L.down;
}

// Consumers: one stage.  Returns false once the CTA is aborting.
template <int B, int D, bool MOE, int VAR>
__device__ __noinline__ bool consume_stage(const Params& p, Ctx& cx, int kind, int l, int s,
                                           RingPos& rp, bool fused) {
  constexpr bool KV8 = (VAR & 1) != 0;   // e4m3 KV cache
  constexpr bool W4 = (VAR & 2) != 0;    // NVFP4 weights
  const unsigned G = static_cast<unsigned>(p.G);
  const unsigned S1 = static_cast<unsigned>(p.step_base + s + 1);
  const int where = where_code(kind, l, s);
  if (kind == ST_ATTN) {
    consume_attn<B, D, KV8>(p, cx, l, s, rp, fused);
    const bool ab = consumer_sync_any(cx.ctl->abort != 0);
    if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 3);
    return !ab;
  }
  const int ffn_done = p.ffn_fused ? ST_GATEUP : ST_DOWN;   // the stage that completes a layer
  if (kind == ST_DOWN && p.ffn_fused) return true;         // done inside the fused gate/up stage
  if (kind == ST_LM) {
    if (!stage_wait(p, cx, p.cnt + (p.L - 1) * ST_LAYER + ffn_done, G * S1, where, fused)) return false;
    float* hid = (p.hidden_out && cx.c == 0)
                     ? p.hidden_out + static_cast<size_t>(p.hidden_overwrite ? 0 : s) * p.B * p.H
                     : nullptr;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    EpiLM<B> epi{p, s, &bv, &bi};
    bool on_tc = false;
    if constexpr (B == kMaxBatch && !MOE) {
      if (p.tc) {
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
        consume_tc(p, cx, p.lm, rp, where, SRC_RESID, p.x, p.final_norm, hid, epi);
        on_tc = true;
      }
    }
    if (!on_tc) {
      float rn[B];
      load_act<B>(p, cx, p.H, p.resid_fixed ? SRC_FIXED : SRC_RESID, resid_src(p), p.final_norm, hid, SIDE_NONE, s, rn,
                  where);
      if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
      consume_gemv<B, W4>(p, cx, p.lm, rp, where, rn, epi);
    }
    if (cx.lane < B) {
      cx.ctl->redv[cx.warp][cx.lane] = bv;
      cx.ctl->redi[cx.warp][cx.lane] = bi;
    }
    consumer_sync();
    if (cx.tid < B) {
      float v = -INFINITY;
      int ix = 0x7fffffff;
      for (int w = 0; w < kConsumerWarps; ++w) argmax_merge(v, ix, cx.ctl->redv[w][cx.tid], cx.ctl->redi[w][cx.tid]);
      p.lm_val[cx.c * p.B + cx.tid] = v;
      p.lm_idx[cx.c * p.B + cx.tid] = ix;
    }
    consumer_sync();
    if (cx.tid == 0) {
      const unsigned old = release_add(p.cnt + p.cl.lm_arrive, 1u);
      __threadfence();
      cx.ctl->flag = (old == G * S1 - 1u) ? 1 : 0;
    }
    consumer_sync();
    if (cx.ctl->flag) {
      if (cx.warp < B) {
        const int b = cx.warp;
        float v = -INFINITY;
        int ix = 0x7fffffff;
        for (int c2 = cx.lane; c2 < p.G; c2 += 32)
          argmax_merge(v, ix, __ldcg(p.lm_val + c2 * p.B + b), __ldcg(p.lm_idx + c2 * p.B + b));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
          const int i2 = __shfl_xor_sync(0xffffffffu, ix, o);
          argmax_merge(v, ix, v2, i2);
        }
        if (cx.lane == 0) {
          int nxt = p.forced ? p.forced[static_cast<size_t>(s) * p.B + b] : ix;
          // A token outside [0, V) (all-NaN logits, or a bad forced token)
          // would index past the embedding table: record it and feed 0.
          if (ix < 0 || ix >= p.V || nxt < 0 || nxt >= p.V) {
            raise_error(p, kErrAborted, where_code(ST_LM, 0, s) | (1 << 14));
            if (ix < 0 || ix >= p.V) ix = 0;
            if (nxt < 0 || nxt >= p.V) nxt = 0;
          }
          p.tokens_out[static_cast<size_t>(s) * p.B + b] = ix;
          p.cur_tok[b] = nxt;
          if (p.serve)
            p.serve_tokens_host[static_cast<size_t>((p.serve_step0 + s) % p.serve_cap) * p.B + b] = ix;
        }
      }
      consumer_sync();
      if (p.verify && cx.tid == 0) {
        // accept drafts while the argmax after position pos0[a] is draft a
        int a = 0;
        while (a < p.B - 1 && p.tokens_out[a] == p.draft[a]) ++a;
        p.accept_out[0] = a + 1;                 // the accepted drafts and the bonus token
        p.cur_tok[0] = p.tokens_out[a];           // the next pending token
      }
      if (cx.tid == 0) {
        release_add(p.cnt + p.cl.step_done, 1u);
        if (p.serve) {
          // the step's tokens (written above, ordered by the barrier) before its count, to the host
          __threadfence_system();
          asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p.serve_done_host),
                       "r"(static_cast<unsigned>(p.serve_step0 + s + 1))
                       : "memory");
        }
      }
    }
    const bool ab = consumer_sync_any(cx.ctl->abort != 0);
    if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 3);
    return !ab;
  }
  const LayerParams& L = p.layers[l];
  bool ok = true;
  float rn[B];
  int r0, r1;
  resid_rows<B>(p, cx.c, r0, r1);
  bool on_tc = false;
  if constexpr (B == kMaxBatch && !MOE) {
    if (p.tc) {
      // batch-8 tensor-core stages: same waits, side data and epilogues
      on_tc = true;
      const unsigned* dep;
      unsigned tgt;
      if (kind == ST_QKV) {
        dep = l == 0 ? p.cnt + p.cl.step_done : p.cnt + (l - 1) * ST_LAYER + ffn_done;
        tgt = l == 0 ? S1 - 1u : G * S1;
      } else if (kind == ST_OPROJ) {
        dep = p.cnt + l * ST_LAYER + ST_ATTN;
        tgt = static_cast<unsigned>(p.B * p.nkv) * S1;
      } else if (kind == ST_GATEUP) {
        dep = p.cnt + l * ST_LAYER + ST_OPROJ;
        tgt = G * S1;
      } else {
        dep = p.cnt + l * ST_LAYER + ST_GATEUP;
        tgt = G * S1;
      }
      if (!stage_wait(p, cx, dep, tgt, where, fused)) return false;
      if (kind == ST_QKV) {
        load_side<B>(p, cx, SIDE_ROPE, s, where);
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
        EpiQKV<B, KV8> epi{p, l, s, reinterpret_cast<const float2*>(cx.side + p.side_rope)};
        consume_tc(p, cx, L.qkv, rp, where, l == 0 ? SRC_EMBED : SRC_RESID, p.x, L.attn_norm, nullptr, epi);
      } else if (kind == ST_OPROJ) {
        load_side<B>(p, cx, l == 0 ? SIDE_EMBED : SIDE_RESID, s, where);
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
        EpiResid<B> epi{p, l == 0, cx.side, r0};
        consume_tc(p, cx, L.o, rp, where, SRC_PLAIN, p.o, nullptr, nullptr, epi);
      } else if (kind == ST_GATEUP) {
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
        EpiSwiGLU<B> epi{p};
        consume_tc(p, cx, L.gu, rp, where, SRC_RESID, p.x, L.ffn_norm, nullptr, epi);
      } else {
        load_side<B>(p, cx, SIDE_RESID, s, where);
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
        EpiResid<B> epi{p, false, cx.side, r0};
        consume_tc(p, cx, L.down, rp, where, SRC_PLAIN, p.h, nullptr, nullptr, epi);
      }
    }
  }
  if (!on_tc) switch (kind) {
    case ST_QKV: {
      if (l == 0) {
        ok = stage_wait(p, cx, p.cnt + p.cl.step_done, S1 - 1u, where, fused);
        if (!ok) return false;
        load_act<B>(p, cx, p.H, SRC_EMBED, nullptr, L.attn_norm, nullptr, SIDE_ROPE, s, rn, where);
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
      } else {
        ok = stage_wait(p, cx, p.cnt + (l - 1) * ST_LAYER + ffn_done, G * S1, where, fused);
        if (!ok) return false;
        load_act<B>(p, cx, p.H, p.resid_fixed ? SRC_FIXED : SRC_RESID, resid_src(p), L.attn_norm, nullptr, SIDE_ROPE, s,
                    rn, where);
        if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
      }
      EpiQKV<B, KV8> epi{p, l, s, reinterpret_cast<const float2*>(cx.side + p.side_rope)};
      consume_gemv<B, W4>(p, cx, L.qkv, rp, where, rn, epi);
      break;
    }
    case ST_OPROJ: {
      const unsigned tgt = static_cast<unsigned>(p.B * p.nkv) * S1;
      if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_ATTN, tgt, where, fused)) return false;
      load_act<B>(p, cx, p.nq * p.d, SRC_PLAIN, p.o, nullptr, nullptr, l == 0 ? SIDE_EMBED : SIDE_RESID, s,
                  rn, where);
      if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
      EpiResid<B> epi{p, l == 0, cx.side, r0, p.ffn_fused ? p.y : nullptr};
      consume_gemv<B, W4>(p, cx, L.o, rp, where, rn, epi);
      break;
    }
    case ST_GATEUP: {
      if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_OPROJ, G * S1, where, fused)) return false;
      load_act<B>(p, cx, p.H, SRC_RESID, p.ffn_fused ? p.y : p.x, L.ffn_norm, nullptr, SIDE_NONE, s, rn, where);
      if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
      if constexpr (MOE) {
        if constexpr (B == 1) {
          // router (all E logits in every CTA), routing, then this CTA's groups
          // of the virtual [slot][pair] gate/up space
          EpiRouter<B> er{cx.ctl->logits};
          consume_gemv<B, W4>(p, cx, L.router, rp, where, rn, er, 0, L.router.N >> 1);
          consumer_sync();
          if (cx.warp == 0) moe_route(p, cx, l, s);
          consumer_sync();
          const int ng = p.S * (p.Fe >> 3);
          Mat v = L.egu;
          v.N = 2 * p.S * p.Fe;
          EpiMoeGU<B> eg{p, cx.ctl->route_w};
          consume_gemv<B, W4>(p, cx, v, rp, where, rn, eg, 8 * split_point(cx.c, ng, p.G),
                          8 * split_point(cx.c + 1, ng, p.G));
        }
      } else if (p.ffn_fused) {
        // gate/up into this CTA's h slice, then its columns of W_down, added into x
        const int q0 = split_point(cx.c, p.F, p.G), q1 = split_point(cx.c + 1, p.F, p.G);
        float* hl = reinterpret_cast<float*>(cx.side + p.side_hloc);
        EpiSwiGLULocal<B> epi{hl, p.hloc, q0};
        consume_gemv<B, W4>(p, cx, L.gu, rp, where, rn, epi);
        consumer_sync();
        consume_downT<B>(p, cx, rp, where, q0, q1, hl);
      } else {
        EpiSwiGLU<B> epi{p};
        consume_gemv<B, W4>(p, cx, L.gu, rp, where, rn, epi);
      }
      break;
    }
    default: {  // ST_DOWN
      if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_GATEUP, G * S1, where, fused)) return false;
      if constexpr (!MOE && B >= 2) {   // (batch 1 inputs always fit whole)
        if (p.down_win > 0) {
          if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
          EpiResid<B> epi{p, false, cx.side, r0};
          if (L.down.fp8)
            consume_gemv_win_t<B, true>(p, cx, L.down, rp, where, p.h, s, epi);
          else
            consume_gemv_win_t<B, false>(p, cx, L.down, rp, where, p.h, s, epi);
          break;
        }
      }
      const int K = MOE ? p.S * p.Fe : p.F;
      load_act<B>(p, cx, K, SRC_PLAIN, p.h, nullptr, nullptr, SIDE_RESID, s, rn, where);
      if (cx.tid == 0) trace_stamp(p, s, stage_index(p, kind, l), 2);
      EpiResid<B> epi{p, false, cx.side, r0};
      if constexpr (MOE) {
        // K runs over [slot][expert column]: the producer streams each slot's expert
        Mat v = L.edown;
        v.K = K;
        consume_gemv<B, W4>(p, cx, v, rp, where, rn, epi);
      } else {
        consume_gemv<B, W4>(p, cx, L.down, rp, where, rn, epi);
      }
      break;
    }
  }
  // Every stage's outputs (KV entries, q, x, h) are read later through the
  // async proxy (bulk copies, here or in other CTAs): order this thread's
  // generic writes first.
  fence_proxy_async_global();
  const bool ab = consumer_sync_any(cx.ctl->abort != 0);
  if (cx.tid == 0) {
    trace_stamp(p, s, stage_index(p, kind, l), 3);
    const bool dropped = p.fault_drop_stage == stage_index(p, kind, l) && cx.c == 0 && s == 0;
    if (!dropped) release_add(p.cnt + l * ST_LAYER + kind, 1u);
  }
  return !ab;
}

// ------------------------------------------------------------------ kernels

__device__ __forceinline__ Ctx make_ctx(uint8_t* smem, const Params& p) {
  Ctx cx;
  cx.ring = smem;
  cx.act = reinterpret_cast<float*>(smem + static_cast<size_t>(p.nslot) * kSlotBytes);
  cx.side = smem + static_cast<size_t>(p.nslot) * kSlotBytes + p.act_bytes;
  cx.ctl = reinterpret_cast<SmemCtl*>(cx.side + p.side_bytes);
  cx.c = blockIdx.x;
  cx.tid = threadIdx.x;
  cx.warp = threadIdx.x >> 5;
  cx.lane = threadIdx.x & 31;
  cx.act_phase = 0;
  cx.acc_phase = 0;
  cx.bop_phase = 0;
  return cx;
}

__device__ __forceinline__ void init_ring(const Params& p, Ctx& cx) {
#ifdef XLPK_DEBUG_POISON
  // Debug build: fill the ring and the activation region with NaN bit
  // patterns so that a read of shared memory nobody wrote shows up as NaN.
  {
    uint32_t* w = reinterpret_cast<uint32_t*>(cx.ring);
    const int n = (p.nslot * kSlotBytes + p.act_bytes) >> 2;
    for (int i = cx.tid; i < n; i += kThreads) w[i] = 0xffffffffu;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
#endif
  if (cx.tid == 0) {
    for (int i = 0; i < p.nslot; ++i) {
      mbar_init(smem_addr(&cx.ctl->full[i]), 1);
      mbar_init(smem_addr(&cx.ctl->empty[i]), kConsumerWarps);
    }
    mbar_init(smem_addr(&cx.ctl->act_bar), 1);
    mbar_init(smem_addr(&cx.ctl->acc_bar), 1);
    mbar_init(smem_addr(&cx.ctl->bop_bar), 1);
    mbar_init(smem_addr(&cx.ctl->fin_bar), 1);
    cx.ctl->abort = 0;
    cx.ctl->flag = 0;
    cx.ctl->route_seq = 0;
    for (int k = 0; k < 8; ++k) cx.ctl->tacc[k] = 0;
    fence_barrier_init();
  }
  __syncthreads();
}

// Producer epilogue: wait until every issued copy has landed so the CTA's
// shared memory is not released under an in-flight bulk copy.
static __device__ void drain_ring(const Params& p, Ctx& cx, const RingPos& rp, int issued) {
  if (issued <= 0) return;
  const int n = min(issued, p.nslot);
  RingPos q = rp;
  for (int k = 0; k < n; ++k) {
    // step back one slot
    if (q.slot == 0) {
      q.slot = p.nslot - 1;
      q.phase ^= 1u;
    } else {
      --q.slot;
    }
    copy_wait(p, smem_addr(&cx.ctl->full[q.slot]), q.phase);
  }
}

// ------------------------------------------------------------------ producer

// One tile of the CTA's stream: one contiguous global range (a packed weight
// tile) or two (the K rows and V rows of an attention chunk, the V rows landing
// at the slot's second half).
struct Tile {
  const uint8_t* src;   // GEMV: packed tile
  int y;                // attention: first cache row of the chunk (tensor-map row)
  int rows;             // attention: positions of the chunk that exist (<= chunk size)
  uint32_t bytes;       // bytes landing in the slot
  bool attn;
  int stage;            // stage_index
  int layer;
  int step;
};

// A position in the CTA's static schedule: steps x (layers x 5 stages + LM).
// The producer runs two: the copy cursor (tiles into the ring) and, ahead of
// it, the prefetch cursor (the same tiles into L2).
template <int B>
struct Cursor {
  int s, l, kind;
  bool open;           // the current stage's range has been set up
  bool one_stage;      // kernel-per-op launch: only one stage
  bool done;
  int a, a_end;        // GEMV: next pair of the CTA's span / span end; attention: item range;
                       // MoE gate/up experts: next virtual group / end
  int kc, nkc, KC;
  int esz;             // bytes per weight element of the current matrix
  int trow;            // packed bytes per row of one tile (codes/values + FP8 scales)
  const uint8_t* src;  // GEMV: next tile
  int phase;           // MoE gate/up: 0 router, 1 experts
  int slot, grp;       // MoE down: slot of the next tile, group index within the CTA's span
  AttnPlan<B> ap;
};

template <int B>
__device__ __forceinline__ void cursor_start(Cursor<B>& cu, int s, int l, int kind, bool one) {
  cu.s = s;
  cu.l = l;
  cu.kind = kind;
  cu.open = false;
  cu.one_stage = one;
  cu.done = false;
}

template <int B>
__device__ __forceinline__ void cursor_next_stage(const Params& p, Cursor<B>& cu) {
  cu.open = false;
  if (cu.one_stage) {
    cu.done = true;
  } else if (cu.kind == ST_LM) {
    cu.kind = 0;
    cu.l = 0;
    if (++cu.s >= p.n_steps) cu.done = true;
  } else {
    ++cu.kind;
    if (cu.kind == ST_DOWN && p.ffn_fused) ++cu.kind;   // done inside the fused gate/up stage
    if (cu.kind == ST_LAYER) {
      cu.kind = 0;
      if (++cu.l == p.L) {
        cu.kind = ST_LM;
        cu.l = 0;
      }
    }
  }
}

enum CursorResult : int { CUR_DONE = 0, CUR_TILE = 1, CUR_BLOCKED = 2, CUR_RUN = 3, CUR_REQ = 4 };

// A dense GEMV stage of one CTA is one contiguous byte range: n1 tiles of b1
// bytes (full groups of 8 row pairs), then n2 tiles of b2 bytes (the last,
// partial group).  The producer drains it from registers.
struct Run {
  const uint8_t* src;
  int n1, n2;
  uint32_t b1, b2;
  int stage, layer, step;
};

template <int B, bool MOE, int VAR>
__device__ int cursor_next(const Params& p, int c, const SmemCtl* ctl, Cursor<B>& cu, Tile& t, Run* run) {
  constexpr bool KV8 = (VAR & 1) != 0;   // e4m3 KV cache
  while (!cu.done) {
    if (p.serve && !cu.open && !cu.one_stage && cu.kind == ST_QKV && cu.l == 0) {
      // serve mode: a step's tiles are streamed once the step is requested
      const int st = serve_state(p, cu.s);
      if (st < 0) {
        cu.done = true;
        break;
      }
      if (st == 0) return CUR_REQ;
    }
    const bool moe = MOE && (cu.kind == ST_GATEUP || cu.kind == ST_DOWN);
    if (!cu.open) {
      cu.open = true;
      cu.esz = p.esz;
      if (cu.kind == ST_ATTN) {
        attn_plan<B>(p, cu.s, cu.ap);
        attn_cta_items<B>(p, cu.ap, c, cu.a, cu.a_end);
      } else if (moe && cu.kind == ST_GATEUP) {
        // the router first (every CTA streams all of it), then the CTA's groups
        // of the virtual [slot][pair] space
        const Mat& r = p.layers[cu.l].router;
        cu.phase = 0;
        cu.a = 0;
        cu.a_end = r.N >> 1;
        cu.kc = 0;
        cu.nkc = r.K / r.KC;
        cu.KC = r.KC;
        cu.esz = 2;
        cu.trow = packed_row_bytes(r, r.KC);
        cu.src = r.packed;
      } else if (moe) {   // MoE down: the CTA's output rows, every slot's expert in turn
        const Mat& m = p.layers[cu.l].edown;
        cu.a = split_point(c, p.H >> 1, p.G);
        cu.a_end = split_point(c + 1, p.H >> 1, p.G);
        cu.kc = 0;
        cu.nkc = m.K / m.KC;
        cu.KC = m.KC;
        cu.slot = 0;
        cu.grp = 0;
      } else if (B == kMaxBatch && p.tc) {
        // batch-8 tensor-core tiles: the CTA's 8-row units, runs per K window
        const Mat& m = (cu.kind == ST_LM) ? p.lm : stage_mat(p.layers[cu.l], cu.kind);
        const int U = m.N >> 3;
        const int u0 = split_point(c, U, p.G), u1 = split_point(c + 1, U, p.G);
        cu.a = 4 * u0;
        cu.a_end = 4 * u1;
        cu.kc = 0;
        cu.phase = 0;
        cu.src = m.packed + static_cast<size_t>(8) * u0 * tc_row_bytes(m.K, m.fp8);
      } else {
        const Mat& m = (cu.kind == ST_LM) ? p.lm : stage_mat(p.layers[cu.l], cu.kind);
        const int NP = m.N >> 1;
        cu.a = split_point(c, NP, p.G);
        cu.a_end = split_point(c + 1, NP, p.G);
        cu.kc = 0;
        cu.nkc = m.K / m.KC;
        cu.KC = m.KC;
        cu.trow = packed_row_bytes(m, m.KC);
        cu.src = m.packed + static_cast<size_t>(2) * cu.a * packed_row_bytes(m, m.K);
        cu.phase = 0;
      }
    }
    t.stage = stage_index(p, cu.kind, cu.l);
    t.layer = cu.l;
    t.step = cu.s;
    t.attn = false;
    if (cu.kind == ST_ATTN) {
      if (cu.a < cu.a_end) {   // every chunk is one tile (K and V boxes)
        int b, g, j, nch, base;
        attn_item<B>(p, cu.ap, cu.a, b, g, j, nch, base);
        ++cu.a;
        bool ok;
        t.y = static_cast<int>(kv_row(p, cu.l, b, g, j * p.attn_pos_per_tile, ok) / p.d);
        if (!ok) raise_error(p, kErrBadPage, where_code(ST_ATTN, cu.l, cu.s));   // row 0 is read instead
        t.rows = min(p.attn_pos_per_tile, p.pos0[b] + cu.s + 1 - j * p.attn_pos_per_tile);
        t.src = nullptr;
        t.bytes = KV8 ? kTileBytes / 2 : kTileBytes;   // two boxes of P x d entries
        t.attn = true;
        return CUR_TILE;
      }
    } else if (moe && cu.kind == ST_GATEUP && cu.phase == 1) {
      if (cu.a < cu.a_end) {
        const LayerParams& L = p.layers[cu.l];
        const int gpe = p.Fe >> 3;                     // groups of 8 pairs per expert
        const int slot = cu.a / gpe, grp = cu.a - slot * gpe;
        if (slot >= p.nsh && ctl->route_seq != route_want(p, cu.s, cu.l)) return CUR_BLOCKED;
        const int ex = slot < p.nsh ? p.E + slot : ctl->route_exp[slot];
        const uint32_t tb = 2u * kPairsPerTile * cu.KC * cu.esz;
        t.bytes = tb;
        t.src = L.egu.packed + ex * L.egu_stride + (static_cast<size_t>(grp) * cu.nkc + cu.kc) * tb;
        if (++cu.kc == cu.nkc) {
          cu.kc = 0;
          ++cu.a;
        }
        return CUR_TILE;
      }
    } else if (moe && cu.kind == ST_DOWN) {
      if (cu.a < cu.a_end) {
        if (ctl->route_seq != route_want(p, cu.s, cu.l)) return CUR_BLOCKED;
        const LayerParams& L = p.layers[cu.l];
        const int gp = min(kPairsPerTile, cu.a_end - cu.a);
        const int ex = ctl->route_exp[cu.slot];
        const int a0 = split_point(c, p.H >> 1, p.G);
        t.bytes = 2u * gp * cu.KC * cu.esz;
        t.src = L.edown.packed + ex * L.edown_stride +
                (static_cast<size_t>(2) * a0 * p.Fe + static_cast<size_t>(cu.grp) * 2 * kPairsPerTile * p.Fe) *
                    cu.esz +
                static_cast<size_t>(cu.kc) * t.bytes;
        if (++cu.kc == cu.nkc) {
          cu.kc = 0;
          if (++cu.slot == p.S) {
            cu.slot = 0;
            ++cu.grp;
            cu.a += kPairsPerTile;
          }
        }
        return CUR_TILE;
      }
    } else if (!MOE && B == kMaxBatch && p.tc && cu.a < cu.a_end) {
      // batch-8 tensor-core stage: per K window one run, the full 128-row
      // M-tiles' tiles then the last M-tile's (params.h: tile geometry)
      const Mat& m = (cu.kind == ST_LM) ? p.lm : stage_mat(p.layers[cu.l], cu.kind);
      const int win = tc_window(p.tc_win, m.K);
      const int fp8 = m.fp8, bc = tc_box_cols(fp8), kbox = tc_kbox(m.K, win, fp8);
      const int R = 2 * (cu.a_end - cu.a), w = cu.phase;
      const int k0 = w * win, Kw = win > 0 ? min(win, m.K - k0) : m.K;
      const int rl = R - 128 * ((R - 1) >> 7);    // rows of the last M-tile
      const int nfull = (R - rl) >> 7;
      const int nb1 = tc_nb(128, kbox, fp8), nbl = tc_nb(rl, kbox, fp8);
      run->src = cu.src + static_cast<size_t>(w) * R * tc_row_bytes(win, fp8);
      if (rl == 128) {
        run->n1 = (nfull + 1) * ((Kw / bc) / nb1);
        run->n2 = 0;
      } else {
        run->n1 = nfull * ((Kw / bc) / nb1);
        run->n2 = (Kw / bc) / nbl;
      }
      run->b1 = static_cast<uint32_t>(tc_tile_bytes(128, nb1, fp8));
      run->b2 = static_cast<uint32_t>(tc_tile_bytes(rl, nbl, fp8));
      run->stage = t.stage;
      run->layer = t.layer;
      run->step = t.step;
      ++cu.phase;
      if (win == 0 || cu.phase * win >= m.K) cu.a = cu.a_end;
      return CUR_RUN;
    } else if (!MOE && B >= 2 && cu.kind == ST_DOWN && p.down_win > 0 && cu.a < cu.a_end) {
      // K-windowed down projection: one run per window (its tiles: the full
      // groups' chunks of the window, then the partial group's); cu.phase
      // counts the windows
      const int np = cu.a_end - cu.a;
      const int cw = p.down_win / cu.KC, w = cu.phase;
      const int cww = min(cw, cu.nkc - w * cw);
      run->src = cu.src + static_cast<size_t>(2) * np * cw * w * cu.trow;
      run->n1 = (np / kPairsPerTile) * cww;
      run->b1 = 2u * kPairsPerTile * cu.trow;
      run->n2 = (np % kPairsPerTile) ? cww : 0;
      run->b2 = 2u * (np % kPairsPerTile) * cu.trow;
      run->stage = t.stage;
      run->layer = t.layer;
      run->step = t.step;
      if (++cu.phase * cw >= cu.nkc) cu.a = cu.a_end;
      return CUR_RUN;
    } else if (cu.a < cu.a_end && !(moe && cu.kind == ST_GATEUP) && cu.kc == 0) {
      // a whole dense stage (the MoE router goes tile by tile)
      const int np = cu.a_end - cu.a;
      run->src = cu.src;
      run->n1 = (np / kPairsPerTile) * cu.nkc;
      run->b1 = 2u * kPairsPerTile * cu.trow;
      run->n2 = (np % kPairsPerTile) ? cu.nkc : 0;
      run->b2 = 2u * (np % kPairsPerTile) * cu.trow;
      run->stage = t.stage;
      run->layer = t.layer;
      run->step = t.step;
      cu.a = cu.a_end;
      return CUR_RUN;
    } else if (cu.a < cu.a_end) {
      const int gp = min(kPairsPerTile, cu.a_end - cu.a);
      t.bytes = 2u * gp * cu.trow;
      t.src = cu.src;
      cu.src += t.bytes;
      if (++cu.kc == cu.nkc) {
        cu.kc = 0;
        cu.a += kPairsPerTile;
      }
      return CUR_TILE;
    } else if (!MOE && p.ffn_fused && cu.kind == ST_GATEUP && cu.phase == 0) {
      // fused FFN: after the gate/up run, this CTA's rows of W_down^T (one run)
      const int j0 = split_point(c, p.F, p.G), j1 = split_point(c + 1, p.F, p.G);
      const int nj = j1 - j0;
      cu.phase = 1;
      if (nj > 0) {
        const uint32_t colb = static_cast<uint32_t>(p.H) * 2u;
        run->src = p.layers[cu.l].downT.packed + static_cast<size_t>(j0) * colb;
        run->n1 = nj / p.jt;
        run->b1 = static_cast<uint32_t>(p.jt) * colb;
        run->n2 = (nj % p.jt) ? 1 : 0;
        run->b2 = static_cast<uint32_t>(nj % p.jt) * colb;
        run->stage = t.stage;
        run->layer = t.layer;
        run->step = t.step;
        return CUR_RUN;
      }
      continue;
    } else if (moe && cu.kind == ST_GATEUP && cu.phase == 0) {
      // router done: the experts' gate/up groups of this CTA
      const Mat& m = p.layers[cu.l].egu;
      const int ng = p.S * (p.Fe >> 3);
      cu.phase = 1;
      cu.a = split_point(c, ng, p.G);
      cu.a_end = split_point(c + 1, ng, p.G);
      cu.kc = 0;
      cu.nkc = m.K / m.KC;
      cu.KC = m.KC;
      cu.esz = p.esz;
      continue;
    }
    cursor_next_stage<B>(p, cu);
  }
  return CUR_DONE;
}

__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Bounded wait of the producer for its CTA's routing of (step, layer).
static __device__ __noinline__ bool route_wait(const Params& p, SmemCtl* ctl, int want, int where) {
  const uint64_t t0 = globaltimer();
  while (ctl->route_seq != want) {
    if (ctl->abort) return false;
    if (ld_volatile(p.abort_flag)) {
      ctl->abort = 1;
      return false;
    }
    if (static_cast<long long>(globaltimer() - t0) > 2 * p.spin_limit_ns) {
      raise_error(p, kErrTimeout, where);
      ctl->abort = 1;
      return false;
    }
    __nanosleep(32);
  }
  __threadfence_block();   // the table was written before route_seq
  return true;
}

// The producer (one thread): copy cursor -> ring, prefetch cursor -> L2,
// `p.l2_prefetch_bytes` ahead.  Weights do not depend on activations, so both
// run ahead of the consumers across stage boundaries; only attention chunks
// wait for the previous step's KV write of their layer.
template <int B, bool MOE, int VAR>
__device__ void producer_main(const Params& p, Ctx& cx, int kind0, int l0, int s0, bool fused) {
  constexpr bool KV8 = (VAR & 1) != 0;   // e4m3 KV cache
  RingPos rp;
  const uint64_t pol = evict_first_policy();
  Cursor<B> cc, pc;
  cursor_start<B>(cc, s0, l0, kind0, !fused);
  cursor_start<B>(pc, s0, l0, kind0, !fused);
  long long ahead = 0;
  bool pc_live = true;
  int cur_stage = -1, cur_step = -1;
  // The copy cursor's current tile and dense run live in scalars (registers);
  // only the slow path (stage changes, attention, MoE) goes through the
  // memory-resident Cursor/Tile/Run structures.
  Tile t, tp;
  Run nr, prun;
  const uint8_t* r_src = nullptr;
  int r_n1 = 0, r_n2 = 0;
  uint32_t r_b1 = 0, r_b2 = 0;
  int r_stage = 0, r_layer = 0, r_step = 0;
  const uint8_t* pf_src = nullptr;   // the prefetch cursor's current dense range
  long long pf_left = 0;
  for (;;) {
    const uint8_t* t_src;
    uint32_t tb;
    bool t_attn = false;
    int t_stage, t_layer, t_step, t_y = 0;
    if (r_n1 + r_n2 == 0) {
      int r = cursor_next<B, MOE, VAR>(p, cx.c, cx.ctl, cc, t, &nr);
      while (r == CUR_REQ) {
        // serve mode: the next step is not requested yet (bounded wait)
        if (!serve_gate(p, cx.ctl, cc.s, false) && serve_state(p, cc.s) >= 0) break;
        r = cursor_next<B, MOE, VAR>(p, cx.c, cx.ctl, cc, t, &nr);
      }
      if (r == CUR_REQ) break;
      if (r == CUR_BLOCKED) {
        // the next tile is an expert chosen by this CTA's own consumers: wait
        // (bounded) until they publish the layer's routing
        if (!route_wait(p, cx.ctl, route_want(p, cc.s, cc.l), where_code(cc.kind, cc.l, cc.s) | (1 << 15))) break;
        r = cursor_next<B, MOE, VAR>(p, cx.c, cx.ctl, cc, t, &nr);
      }
      if (r == CUR_RUN) {
        r_src = nr.src;
        r_n1 = nr.n1;
        r_n2 = nr.n2;
        r_b1 = nr.b1;
        r_b2 = nr.b2;
        r_stage = nr.stage;
        r_layer = nr.layer;
        r_step = nr.step;
      } else if (r != CUR_TILE) {
        break;
      }
    }
    if (r_n1 + r_n2 > 0) {   // next tile of the dense run
      t_src = r_src;
      tb = r_n1 ? r_b1 : r_b2;
      if (r_n1) --r_n1; else --r_n2;
      r_src += tb;
      t_stage = r_stage;
      t_layer = r_layer;
      t_step = r_step;
    } else {
      t_src = t.src;
      tb = t.bytes;
      t_attn = t.attn;
      t_stage = t.stage;
      t_layer = t.layer;
      t_step = t.step;
      t_y = t.y;
    }
    ahead -= tb;
    while (pc_live && ahead < p.l2_prefetch_bytes) {
      if (pf_left > 0) {   // dense range: prefetch in tile-sized pieces
        const uint32_t nb = static_cast<uint32_t>(min(pf_left, static_cast<long long>(kTileBytes)));
        prefetch_l2(pf_src, nb);
        pf_src += nb;
        pf_left -= nb;
        ahead += nb;
        continue;
      }
      const int pr = cursor_next<B, MOE, VAR>(p, cx.c, cx.ctl, pc, tp, &prun);
      if (pr == CUR_BLOCKED || pr == CUR_REQ) break;   // resume once the routing / the request is known
      if (pr == CUR_RUN) {
        pf_src = prun.src;
        pf_left = static_cast<long long>(prun.n1) * prun.b1 + static_cast<long long>(prun.n2) * prun.b2;
        continue;
      }
      pc_live = pr == CUR_TILE;
      if (!pc_live) break;
      if (!tp.attn) {
        prefetch_l2(tp.src, tp.bytes);
      } else {
        // the chunk's existing K and V rows (contiguous, 16-byte multiples);
        // L2 is the coherence point, so a row rewritten later is still read fresh
        constexpr int esz = KV8 ? 1 : 2;
        const size_t off = static_cast<size_t>(tp.y) * p.d * esz;
        const uint32_t nb = static_cast<uint32_t>(tp.rows) * p.d * esz;
        prefetch_l2((KV8 ? p.kc8 : reinterpret_cast<const uint8_t*>(p.kc)) + off, nb);
        prefetch_l2((KV8 ? p.vc8 : reinterpret_cast<const uint8_t*>(p.vc)) + off, nb);
      }
      ahead += tp.bytes;
    }
    if (t_stage != cur_stage || t_step != cur_step) {
      if (cur_stage >= 0) trace_stamp(p, cur_step, cur_stage, 5);
      cur_stage = t_stage;
      cur_step = t_step;
      trace_stamp(p, t_step, t_stage, 4);
      if (t_attn) {
        // KV rows up to pos-1 were written by this layer's QKV stage of earlier
        // steps (or before the launch); make sure the previous step's write is
        // complete before reading it through the async proxy.
        if (fused) {
          // (verify: this step's rows of the sequences before this one, too)
          const unsigned target =
              static_cast<unsigned>(p.G) * static_cast<unsigned>(p.step_base + t_step + (p.verify ? 1 : 0));
          const int where = where_code(ST_ATTN, t_layer, t_step) | (1 << 15);
          if (!counter_wait(p, cx.ctl, p.cnt + t_layer * ST_LAYER + ST_QKV, target, where)) break;
        }
        fence_proxy_async_global();
      }
    }
    const uint32_t eb = smem_addr(&cx.ctl->empty[rp.slot]);
    // A full ring only means the consumers are waiting on a dependency; give
    // their own (bounded) wait the chance to time out first, so the reported
    // failure names the dependency rather than this stall.
    if (!mbar_try_wait(eb, rp.phase ^ 1u) &&
        !ring_wait_slow(p, cx.ctl, eb, rp.phase ^ 1u, where_code(t_stage % ST_LAYER, t_layer, t_step) | (1 << 15), 2))
      break;
    const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
    mbar_expect_tx(fb, tb);
    const uint32_t dst = smem_addr(cx.ring + static_cast<size_t>(rp.slot) * kSlotBytes);
    if (KV8 && t_attn) {
      // e4m3 chunk: one box of P rows x d bytes each for K and V
      tma_load_2d(dst, &p.tmap_k, 0, t_y, fb, pol);
      tma_load_2d(dst + 8192, &p.tmap_v, 0, t_y, fb, pol);
    } else if (t_attn) {
      const int box = p.attn_pos_per_tile * 128;
      for (int x = 0; x < p.d; x += 64) {
        tma_load_2d(dst + (x >> 6) * box, &p.tmap_k, x, t_y, fb, pol);
        tma_load_2d(dst + kTileBytes / 2 + (x >> 6) * box, &p.tmap_v, x, t_y, fb, pol);
      }
    } else {
      bulk_g2s(dst, t_src, tb, fb, pol);
    }
    rp.next(p.nslot);
  }
  if (cur_stage >= 0) trace_stamp(p, cur_step, cur_stage, 5);
  // Every slot's most recent copy must have landed before the CTA may exit.
  drain_ring(p, cx, rp, p.nslot);
}

template <int B, int D, bool MOE, int VAR>
__device__ void consumer_main(const Params& p, Ctx& cx, int kind0, int l0, int s0, bool fused) {
  RingPos rp;
  if (fused) {
    for (int s = 0; s < p.n_steps; ++s) {
      if (p.serve) {
        // serve mode: run step s only once the host has asked for it
        const bool go = cx.tid == 0 ? serve_gate(p, cx.ctl, s, cx.c == 0) : true;
        if (consumer_sync_any(!go)) return;
      }
      for (int l = 0; l < p.L; ++l)
        for (int k = 0; k < ST_LAYER; ++k)
          if (!consume_stage<B, D, MOE, VAR>(p, cx, k, l, s, rp, true)) return;
      if (!consume_stage<B, D, MOE, VAR>(p, cx, ST_LM, 0, s, rp, true)) return;
    }
  } else {
    consume_stage<B, D, MOE, VAR>(p, cx, kind0, l0, s0, rp, false);
  }
}

// The persistent engine: one launch decodes p.n_steps tokens.
// Batch-8 tensor-core stages: consumer warp 0 allocates the CTA's accumulator
// columns before the first stage and frees them after the last (every consumer
// leaves consumer_main at the same point, abort included).
template <int B>
__device__ __forceinline__ void tc_open(const Params& p, Ctx& cx) {
  if constexpr (B == kMaxBatch) {
    if (!p.tc) return;
    if (cx.warp == 0) tc_alloc(smem_addr(&cx.ctl->tmem_base), static_cast<uint32_t>(p.tc_cols));
    tc_fence_before();
    consumer_sync();
    tc_fence_after();
  }
}
template <int B>
__device__ __forceinline__ void tc_close(const Params& p, Ctx& cx) {
  if constexpr (B == kMaxBatch) {
    if (!p.tc) return;
    if (cx.warp == 4 && cx.lane == 0) {
      // MMAs may still be in flight after an abort: free the columns only once
      // every one this thread issued has completed (bounded)
      tc_commit(smem_addr(&cx.ctl->fin_bar));
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_addr(&cx.ctl->fin_bar), 0) &&
             static_cast<long long>(globaltimer() - t0) < 2 * p.spin_limit_ns) {
      }
    }
    tc_fence_before();
    consumer_sync();
    if (cx.warp == 0) {
      tc_fence_after();
      tc_dealloc(cx.ctl->tmem_base, static_cast<uint32_t>(p.tc_cols));
    }
  }
}

template <int B, int D, bool MOE, int VAR>
__global__ void __launch_bounds__(kThreads, 1) engine_persistent(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctx cx = make_ctx(smem, p);
  init_ring(p, cx);
  if (cx.warp == kConsumerWarps) {
    if (cx.lane == 0) producer_main<B, MOE, VAR>(p, cx, 0, 0, 0, true);
    __syncwarp();
  } else {
    tc_open<B>(p, cx);
    consumer_main<B, D, MOE, VAR>(p, cx, 0, 0, 0, true);
    tc_close<B>(p, cx);
  }
}

// Kernel-per-op baseline: one launch runs one stage (same tiles, no waits).
template <int B, int D, bool MOE, int VAR>
__global__ void __launch_bounds__(kThreads, 1) engine_stage(const __grid_constant__ Params p, int kind,
                                                            int layer, int step) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctx cx = make_ctx(smem, p);
  if (MOE && kind == ST_DOWN && cx.tid < p.S) {
    // the routing was computed by the gate/up launch: take CTA 0's record
    cx.ctl->route_exp[cx.tid] = p.route_exp[layer * p.S + cx.tid];
    cx.ctl->route_w[cx.tid] = p.route_w[layer * p.S + cx.tid];
  }
  init_ring(p, cx);
  if (MOE && kind == ST_DOWN) {
    if (cx.tid == 0) cx.ctl->route_seq = route_want(p, step, layer);
    __syncthreads();
  }
  if (cx.warp == kConsumerWarps) {
    if (cx.lane == 0) producer_main<B, MOE, VAR>(p, cx, kind, layer, step, false);
    __syncwarp();
  } else {
    tc_open<B>(p, cx);
    consumer_main<B, D, MOE, VAR>(p, cx, kind, layer, step, false);
    tc_close<B>(p, cx);
  }
}

}  // namespace xlpk
