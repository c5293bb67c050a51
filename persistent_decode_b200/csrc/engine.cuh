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
#include <stdint.h>

#include "params.h"

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
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
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
  volatile int abort;
  int flag;
  int pad[2];
  float red[kConsumerWarps][kMaxBatch];
  int redi[kConsumerWarps][kMaxBatch];
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
  SmemCtl* ctl;
  int c;
  int warp;
  int lane;
  int tid;
};

enum ErrCode : int { kErrNone = 0, kErrTimeout = -6, kErrAborted = -7 };

__device__ __forceinline__ void raise_error(const Params& p, int code, int where) {
  if (atomicCAS(p.status, 0, code) == 0) {
    p.status[1] = where;
    p.status[2] = blockIdx.x;
  }
  atomicExch(p.abort_flag, 1);
}

__device__ __forceinline__ int where_code(int kind, int layer, int step) {
  return (step << 16) | ((layer & 0xff) << 8) | (kind & 0xff);
}

// Bounded wait on a ring barrier phase.  Returns false (and marks the CTA
// aborted) if the global abort flag is raised or the time limit passes.
__device__ __noinline__ bool ring_wait_slow(const Params& p, SmemCtl* ctl, uint32_t bar,
                                            uint32_t parity, int where) {
  const uint64_t t0 = globaltimer();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (ctl->abort) return false;
    if ((it & 31u) == 0) {
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

__device__ __forceinline__ bool ring_wait(const Params& p, SmemCtl* ctl, uint32_t bar,
                                          uint32_t parity, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  return ring_wait_slow(p, ctl, bar, parity, where);
}

// Bounded wait (one thread) until *cnt >= target (wrap-safe).
__device__ __noinline__ bool counter_wait_slow(const Params& p, SmemCtl* ctl, const unsigned* cnt,
                                               unsigned target, int where) {
  const uint64_t t0 = globaltimer();
  for (unsigned it = 1;; ++it) {
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
  if (fused && cx.tid == 0) {
    if (!counter_wait(p, cx.ctl, cnt, target, where)) cx.ctl->abort = 1;
  }
  consumer_sync();
  return !cx.ctl->abort;
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

__device__ __forceinline__ uint16_t f2bf(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
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

// Activation vector [B][K] staged in shared memory as two fp32 planes so that
// lane-consecutive 16-byte reads of 8-element weight vectors are conflict-free:
//   plane 0: float4 [B][K/8] = elements 8v..8v+3,  plane 1: elements 8v+4..8v+7.
__device__ __forceinline__ int act_index(int b, int k, int B, int nvK) {
  const int v = k >> 3, e = k & 7;
  return ((((e >> 2) * B + b) * nvK + v) << 2) + (e & 3);
}

enum ActSrc : int { SRC_RESID = 0, SRC_EMBED = 1, SRC_PLAIN = 2 };

// Load the stage input into shared memory.  With `gain`, apply RMSNorm:
// v * rsqrt(mean(v^2) + eps) * gain.  `hidden_dbg` (LM stage, CTA 0) receives
// the raw residual.
template <int B>
__device__ void load_act(const Params& p, Ctx& cx, int K, ActSrc src, const float* gsrc,
                         const float* gain, float* hidden_dbg) {
  const int nvK = K >> 3;
  float ss[B];
  int tok[B];
#pragma unroll
  for (int b = 0; b < B; ++b) {
    ss[b] = 0.f;
    tok[b] = (src == SRC_EMBED) ? __ldcg(p.cur_tok + b) : 0;
  }
  for (int k = cx.tid; k < K; k += kConsumerThreads) {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float v;
      if (src == SRC_EMBED) {
        v = __uint_as_float(static_cast<uint32_t>(p.embed[static_cast<size_t>(tok[b]) * K + k]) << 16);
      } else {
        v = __ldcg(gsrc + static_cast<size_t>(b) * K + k);
      }
      if (hidden_dbg) hidden_dbg[static_cast<size_t>(b) * K + k] = v;
      ss[b] = fmaf(v, v, ss[b]);
      cx.act[act_index(b, k, B, nvK)] = v;
    }
  }
  if (gain) {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const float s = warp_sum(ss[b]);
      if (cx.lane == 0) cx.ctl->red[cx.warp][b] = s;
    }
    consumer_sync();
    float r[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) s += cx.ctl->red[w][b];
      r[b] = rsqrtf(s / static_cast<float>(K) + p.eps);
    }
    for (int k = cx.tid; k < K; k += kConsumerThreads) {
      const float g = __ldg(gain + k);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float& a = cx.act[act_index(b, k, B, nvK)];
        a = a * r[b] * g;
      }
    }
  }
  consumer_sync();
}

// ------------------------------------------------------------------ GEMV stages

// Producer side of one GEMV stage: the CTA's span, tile by tile.
__device__ bool produce_gemv(const Params& p, Ctx& cx, const Mat& m, RingPos& rp, uint64_t pol,
                             int where) {
  const int NP = m.N >> 1;
  const int p0 = split_point(cx.c, NP, p.G), p1 = split_point(cx.c + 1, NP, p.G);
  const int nkc = m.K / m.KC;
  const uint8_t* src = m.packed + static_cast<size_t>(2) * p0 * m.K * p.esz;
  for (int g0 = p0; g0 < p1; g0 += kPairsPerTile) {
    const int gp = min(kPairsPerTile, p1 - g0);
    const uint32_t bytes = 2u * gp * m.KC * p.esz;
    for (int kc = 0; kc < nkc; ++kc) {
      const uint32_t eb = smem_addr(&cx.ctl->empty[rp.slot]);
      if (!ring_wait(p, cx.ctl, eb, rp.phase ^ 1u, where)) return false;
      const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
      mbar_expect_tx(fb, bytes);
      bulk_g2s(smem_addr(cx.ring + static_cast<size_t>(rp.slot) * kSlotBytes), src, bytes, fb, pol);
      src += bytes;
      rp.next(p.nslot);
    }
  }
  return true;
}

// Consumer side: each warp owns one row pair of every tile of a group and
// accumulates it over the group's k-chunks; `epi(pair, acc0, acc1)` runs on
// the reduced sums (identical in every lane).
template <int B, class Epi>
__device__ void consume_gemv(const Params& p, Ctx& cx, const Mat& m, RingPos& rp, int where,
                             Epi& epi) {
  const int NP = m.N >> 1;
  const int p0 = split_point(cx.c, NP, p.G), p1 = split_point(cx.c + 1, NP, p.G);
  const int nkc = m.K / m.KC;
  const int nv = m.KC >> 3;   // 16-byte vectors per row chunk
  const int nvK = m.K >> 3;
  const float4* act_lo = reinterpret_cast<const float4*>(cx.act);
  const float4* act_hi = act_lo + B * nvK;
  for (int g0 = p0; g0 < p1; g0 += kPairsPerTile) {
    const int gp = min(kPairsPerTile, p1 - g0);
    float a0[B], a1[B];
#pragma unroll
    for (int b = 0; b < B; ++b) a0[b] = a1[b] = 0.f;
    for (int kc = 0; kc < nkc; ++kc) {
      const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
      const bool ok = cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where);
      if (ok && cx.warp < gp) {
        const uint4* r0 =
            reinterpret_cast<const uint4*>(cx.ring + static_cast<size_t>(rp.slot) * kSlotBytes) +
            (2 * cx.warp) * nv;
        const uint4* r1 = r0 + nv;
        const int vb = kc * nv;
#pragma unroll 4
        for (int v = cx.lane; v < nv; v += 32) {
          const uint4 w0 = r0[v];
          const uint4 w1 = r1[v];
#pragma unroll
          for (int b = 0; b < B; ++b) {
            const float4 lo = act_lo[b * nvK + vb + v];
            const float4 hi = act_hi[b * nvK + vb + v];
            a0[b] = dot8_bf16(w0, lo, hi, a0[b]);
            a1[b] = dot8_bf16(w1, lo, hi, a1[b]);
          }
        }
      }
      __syncwarp();
      if (cx.lane == 0) mbar_arrive(smem_addr(&cx.ctl->empty[rp.slot]));
      rp.next(p.nslot);
    }
    if (cx.warp < gp) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        a0[b] = warp_sum(a0[b]);
        a1[b] = warp_sum(a1[b]);
      }
      epi(g0 + cx.warp, a0, a1, cx.lane);
    }
  }
}

// QKV epilogue: RoPE on q/k pairs, q -> workspace, bf16 k/v -> cache at pos.
template <int B>
struct EpiQKV {
  const Params& p;
  int l, s;
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
        const float2 cs = __ldg(p.rope + static_cast<size_t>(pos) * half + i);
        const float y0 = r0 * cs.x - r1 * cs.y;
        const float y1 = r0 * cs.y + r1 * cs.x;
        if (isq) {
          float* qd = p.q + (static_cast<size_t>(b) * p.nq + head) * p.d;
          qd[i] = y0;
          qd[i + half] = y1;
        } else {
          uint16_t* kd =
              p.kc + (((static_cast<size_t>(l) * p.B + b) * p.nkv + head) * p.max_seq + pos) * p.d;
          kd[i] = f2bf(y0);
          kd[i + half] = f2bf(y1);
        }
      } else {
        const int pv = pg - hq - hk;
        const int head = pv / half, i2 = (pv - head * half) * 2;
        uint16_t* vd =
            p.vc + (((static_cast<size_t>(l) * p.B + b) * p.nkv + head) * p.max_seq + pos) * p.d;
        const uint32_t packed = static_cast<uint32_t>(f2bf(r0)) | (static_cast<uint32_t>(f2bf(r1)) << 16);
        *reinterpret_cast<uint32_t*>(vd + i2) = packed;
      }
    }
  }
};

// Residual epilogue: x[b][2pg..2pg+1] += (r0, r1); with `embed_base`, x = E[tok] + r.
template <int B>
struct EpiResid {
  const Params& p;
  bool from_embed;
  __device__ void operator()(int pg, const float (&a0)[B], const float (&a1)[B], int lane) const {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (lane != b) continue;
      float2* xp = reinterpret_cast<float2*>(p.x + static_cast<size_t>(b) * p.H) + pg;
      float2 base;
      if (from_embed) {
        const int tok = __ldcg(p.cur_tok + b);
        const uint32_t e = *reinterpret_cast<const uint32_t*>(p.embed + static_cast<size_t>(tok) * p.H + 2 * pg);
        base = make_float2(bf16_lo(e), bf16_hi(e));
      } else {
        base = __ldcg(xp);
      }
      *xp = make_float2(base.x + a0[b], base.y + a1[b]);
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
      p.h[static_cast<size_t>(b) * p.F + pg] = g / (1.f + expf(-g)) * a1[b];
    }
  }
};

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
        float* lo = p.logits_out + (static_cast<size_t>(s) * p.B + b) * p.V + row;
        lo[0] = a0[b];
        lo[1] = a1[b];
      }
    }
  }
};

// ------------------------------------------------------------------ attention

struct AttnPlan {
  int nch[kMaxBatch];
  int base[kMaxBatch];
  int W;
};

__device__ __forceinline__ void attn_plan(const Params& p, int s, AttnPlan& ap) {
  const int P = p.attn_pos_per_tile;
  int w = 0;
  for (int b = 0; b < p.B; ++b) {
    const int T = p.pos0[b] + s + 1;
    ap.nch[b] = (T + P - 1) / P;
    ap.base[b] = w;
    w += p.nkv * ap.nch[b];
  }
  ap.W = w;
}

__device__ __forceinline__ void attn_item(const Params& p, const AttnPlan& ap, int i, int& b, int& g,
                                          int& j) {
  b = 0;
  while (b + 1 < p.B && ap.base[b + 1] <= i) ++b;
  const int r = i - ap.base[b];
  g = r / ap.nch[b];
  j = r - g * ap.nch[b];
}

__device__ __forceinline__ size_t kv_row(const Params& p, int l, int b, int g, int t) {
  return (((static_cast<size_t>(l) * p.B + b) * p.nkv + g) * p.max_seq + t) * p.d;
}

__device__ bool produce_attn(const Params& p, Ctx& cx, int l, int s, RingPos& rp, uint64_t pol,
                             bool fused) {
  AttnPlan ap;
  attn_plan(p, s, ap);
  const int i0 = split_point(cx.c, ap.W, p.G), i1 = split_point(cx.c + 1, ap.W, p.G);
  if (i0 >= i1) return true;
  const int where = where_code(ST_ATTN, l, s) | (1 << 15);
  // Cache rows up to pos-1 were written by this layer's QKV stage of earlier
  // steps (or before the launch).  Make sure the previous step's write is done
  // before reading it through the async proxy.
  if (fused) {
    const unsigned target = static_cast<unsigned>(p.G) * static_cast<unsigned>(p.step_base + s);
    if (!counter_wait(p, cx.ctl, p.cnt + l * ST_LAYER + ST_QKV, target, where)) return false;
  }
  fence_proxy_async_global();
  const int P = p.attn_pos_per_tile;
  const uint32_t vhalf = kSlotBytes / 2;
  for (int i = i0; i < i1; ++i) {
    int b, g, j;
    attn_item(p, ap, i, b, g, j);
    const int T = p.pos0[b] + s + 1;
    const int t_lo = j * P;
    const int n_old = min(t_lo + P, T - 1) - t_lo;
    if (n_old <= 0) continue;
    const uint32_t bytes = static_cast<uint32_t>(n_old) * p.d * 2u;
    const uint32_t eb = smem_addr(&cx.ctl->empty[rp.slot]);
    if (!ring_wait(p, cx.ctl, eb, rp.phase ^ 1u, where)) return false;
    const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
    mbar_expect_tx(fb, 2u * bytes);
    const uint32_t dst = smem_addr(cx.ring + static_cast<size_t>(rp.slot) * kSlotBytes);
    const size_t off = kv_row(p, l, b, g, t_lo);
    bulk_g2s(dst, p.kc + off, bytes, fb, pol);
    bulk_g2s(dst + vhalf, p.vc + off, bytes, fb, pol);
    rp.next(p.nslot);
  }
  return true;
}

// Flash-decoding over this CTA's chunks.  Lanes: grp = lane>>3 picks one of
// 4 positions per warp-round, li = lane&7 owns D/8 of its dims for q.k;
// for p.V each lane owns D/32 consecutive dims.
template <int B, int D>
__device__ void consume_attn(const Params& p, Ctx& cx, int l, int s, RingPos& rp, bool fused) {
  constexpr int NCH = D / 64;   // 8-dim chunks per lane for q.k
  constexpr int DV = D / 32;    // dims per lane for p.V
  AttnPlan ap;
  attn_plan(p, s, ap);
  const int i0 = split_point(cx.c, ap.W, p.G), i1 = split_point(cx.c + 1, ap.W, p.G);
  const int where = where_code(ST_ATTN, l, s);
  const unsigned S1 = static_cast<unsigned>(p.step_base + s + 1);
  if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_QKV, static_cast<unsigned>(p.G) * S1, where, fused))
    return;
  if (i0 >= i1) return;
  const int P = p.attn_pos_per_tile;
  const int GQ = p.group;
  const int grp = cx.lane >> 3, li = cx.lane & 7;
  float* sm_ml = cx.act;                                       // [8][kMaxGroup][2]
  float* sm_o = cx.act + kConsumerWarps * kMaxGroup * 2;       // [8][kMaxGroup][D]

  float qr[kMaxGroup][NCH * 8];
  float m[kMaxGroup], ls[kMaxGroup], oa[kMaxGroup][DV];
  int seg_b = -1, seg_g = -1, seg_first = 0, seg_items = 0;

  for (int i = i0; i < i1; ++i) {
    int b, g, j;
    attn_item(p, ap, i, b, g, j);
    if (b != seg_b || g != seg_g) {
      seg_b = b;
      seg_g = g;
      seg_first = i;
      seg_items = 0;
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        m[h] = -INFINITY;
        ls[h] = 0.f;
#pragma unroll
        for (int e = 0; e < DV; ++e) oa[h][e] = 0.f;
        if (h < GQ) {
          const float* qs = p.q + (static_cast<size_t>(b) * p.nq + g * GQ + h) * D;
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const float4 u = __ldcg(reinterpret_cast<const float4*>(qs + ch * 64 + li * 8));
            const float4 v = __ldcg(reinterpret_cast<const float4*>(qs + ch * 64 + li * 8 + 4));
            qr[h][ch * 8 + 0] = u.x * p.qk_scale_log2;
            qr[h][ch * 8 + 1] = u.y * p.qk_scale_log2;
            qr[h][ch * 8 + 2] = u.z * p.qk_scale_log2;
            qr[h][ch * 8 + 3] = u.w * p.qk_scale_log2;
            qr[h][ch * 8 + 4] = v.x * p.qk_scale_log2;
            qr[h][ch * 8 + 5] = v.y * p.qk_scale_log2;
            qr[h][ch * 8 + 6] = v.z * p.qk_scale_log2;
            qr[h][ch * 8 + 7] = v.w * p.qk_scale_log2;
          }
        } else {
#pragma unroll
          for (int e = 0; e < NCH * 8; ++e) qr[h][e] = 0.f;
        }
      }
    }
    ++seg_items;
    const int T = p.pos0[b] + s + 1;
    const int t_lo = j * P;
    const int npos = min(t_lo + P, T) - t_lo;
    const int n_old = min(t_lo + P, T - 1) - t_lo;
    const uint16_t* sK = nullptr;
    const uint16_t* sV = nullptr;
    bool have_tile = false;
    if (n_old > 0) {
      const uint32_t fb = smem_addr(&cx.ctl->full[rp.slot]);
      have_tile = cx.ctl->abort ? false : ring_wait(p, cx.ctl, fb, rp.phase, where);
      sK = reinterpret_cast<const uint16_t*>(cx.ring + static_cast<size_t>(rp.slot) * kSlotBytes);
      sV = sK + kSlotBytes / 4;
    }
    const uint16_t* gK = p.kc + kv_row(p, l, b, g, T - 1);
    const uint16_t* gV = p.vc + kv_row(p, l, b, g, T - 1);
    for (int r0 = 0; r0 < npos; r0 += 4 * kConsumerWarps) {
      const int r = r0 + cx.warp * 4 + grp;
      const bool valid = r < npos && (r >= n_old || have_tile);
      // q . k for this lane group's position
      float sc[kMaxGroup];
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) sc[h] = 0.f;
      if (valid) {
        const uint16_t* krow = (r < n_old) ? sK + static_cast<size_t>(r) * D : gK;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          uint4 kv;
          if (r < n_old) {
            kv = *reinterpret_cast<const uint4*>(krow + ch * 64 + li * 8);
          } else {
            kv = __ldcg(reinterpret_cast<const uint4*>(krow + ch * 64 + li * 8));
          }
          const float k0 = bf16_lo(kv.x), k1 = bf16_hi(kv.x), k2 = bf16_lo(kv.y), k3 = bf16_hi(kv.y);
          const float k4 = bf16_lo(kv.z), k5 = bf16_hi(kv.z), k6 = bf16_lo(kv.w), k7 = bf16_hi(kv.w);
#pragma unroll
          for (int h = 0; h < kMaxGroup; ++h) {
            float a = sc[h];
            a = fmaf(qr[h][ch * 8 + 0], k0, a);
            a = fmaf(qr[h][ch * 8 + 1], k1, a);
            a = fmaf(qr[h][ch * 8 + 2], k2, a);
            a = fmaf(qr[h][ch * 8 + 3], k3, a);
            a = fmaf(qr[h][ch * 8 + 4], k4, a);
            a = fmaf(qr[h][ch * 8 + 5], k5, a);
            a = fmaf(qr[h][ch * 8 + 6], k6, a);
            a = fmaf(qr[h][ch * 8 + 7], k7, a);
            sc[h] = a;
          }
        }
      }
      float pw[kMaxGroup];
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        float v = sc[h];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        const float sv = valid ? v : -INFINITY;
        float mr = fmaxf(sv, __shfl_xor_sync(0xffffffffu, sv, 8));
        mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, 16));
        const float mn = fmaxf(m[h], mr);
        const float alpha = (mn == -INFINITY) ? 1.f : exp2f(m[h] - mn);
        const float pv = valid ? exp2f(sv - mn) : 0.f;
        float ps = pv + __shfl_xor_sync(0xffffffffu, pv, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
        ls[h] = ls[h] * alpha + ps;
        m[h] = mn;
#pragma unroll
        for (int e = 0; e < DV; ++e) oa[h][e] *= alpha;
        pw[h] = pv;
      }
      // p . V: every lane accumulates its DV dims over the 4 positions
#pragma unroll
      for (int gq = 0; gq < 4; ++gq) {
        const int rr = r0 + cx.warp * 4 + gq;
        const bool vv = rr < npos && (rr >= n_old || have_tile);
        float pg[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) pg[h] = __shfl_sync(0xffffffffu, pw[h], gq * 8);
        if (vv) {
          float vf[DV];
          if (rr < n_old) {
            const uint16_t* vrow = sV + static_cast<size_t>(rr) * D + cx.lane * DV;
            if (DV == 4) {
              const uint2 u = *reinterpret_cast<const uint2*>(vrow);
              vf[0] = bf16_lo(u.x);
              vf[1] = bf16_hi(u.x);
              vf[2] = bf16_lo(u.y);
              vf[3] = bf16_hi(u.y);
            } else {
              const uint32_t u = *reinterpret_cast<const uint32_t*>(vrow);
              vf[0] = bf16_lo(u);
              vf[1] = bf16_hi(u);
            }
          } else {
            const uint16_t* vrow = gV + cx.lane * DV;
            if (DV == 4) {
              const uint2 u = __ldcg(reinterpret_cast<const uint2*>(vrow));
              vf[0] = bf16_lo(u.x);
              vf[1] = bf16_hi(u.x);
              vf[2] = bf16_lo(u.y);
              vf[3] = bf16_hi(u.y);
            } else {
              const uint32_t u = __ldcg(reinterpret_cast<const unsigned int*>(vrow));
              vf[0] = bf16_lo(u);
              vf[1] = bf16_hi(u);
            }
          }
#pragma unroll
          for (int h = 0; h < kMaxGroup; ++h)
#pragma unroll
            for (int e = 0; e < DV; ++e) oa[h][e] = fmaf(pg[h], vf[e], oa[h][e]);
        }
      }
    }
    if (n_old > 0) {
      __syncwarp();
      if (cx.lane == 0) mbar_arrive(smem_addr(&cx.ctl->empty[rp.slot]));
      rp.next(p.nslot);
    }
    // end of a (b, g) segment: merge the 8 warps, publish the partial, and
    // let the CTA that completes the head combine all partials.
    bool seg_end = (i + 1 == i1);
    if (!seg_end) {
      int b2, g2, j2;
      attn_item(p, ap, i + 1, b2, g2, j2);
      seg_end = (b2 != seg_b || g2 != seg_g);
    }
    if (!seg_end) continue;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (cx.lane == 0) {
        sm_ml[(cx.warp * kMaxGroup + h) * 2 + 0] = m[h];
        sm_ml[(cx.warp * kMaxGroup + h) * 2 + 1] = ls[h];
      }
#pragma unroll
      for (int e = 0; e < DV; ++e) sm_o[(cx.warp * kMaxGroup + h) * D + cx.lane * DV + e] = oa[h][e];
    }
    consumer_sync();
    for (int idx = cx.tid; idx < GQ * D; idx += kConsumerThreads) {
      const int h = idx / D, dd = idx - h * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_ml[(w * kMaxGroup + h) * 2]);
      float Ls = 0.f, Os = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = sm_ml[(w * kMaxGroup + h) * 2];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        Ls = fmaf(sm_ml[(w * kMaxGroup + h) * 2 + 1], f, Ls);
        Os = fmaf(sm_o[(w * kMaxGroup + h) * D + dd], f, Os);
      }
      p.part_o[(static_cast<size_t>(seg_first) * GQ + h) * D + dd] = Os;
      if (dd == 0) {
        p.part_ml[(static_cast<size_t>(seg_first) * GQ + h) * 2 + 0] = M;
        p.part_ml[(static_cast<size_t>(seg_first) * GQ + h) * 2 + 1] = Ls;
      }
    }
    consumer_sync();
    unsigned* arrive = p.cnt + p.cl.attn_arrive + (l * p.B + seg_b) * p.nkv + seg_g;
    if (cx.tid == 0) {
      const unsigned old = release_add(arrive, static_cast<unsigned>(seg_items));
      __threadfence();
      cx.ctl->flag = (old + seg_items == static_cast<unsigned>(ap.nch[seg_b])) ? 1 : 0;
    }
    consumer_sync();
    if (cx.ctl->flag) {
      const int ib = ap.base[seg_b] + seg_g * ap.nch[seg_b];
      const int ie = ib + ap.nch[seg_b];
      for (int idx = cx.tid; idx < GQ * D; idx += kConsumerThreads) {
        const int h = idx / D, dd = idx - h * D;
        float M = -INFINITY, Ls = 0.f, Os = 0.f;
        int st = ib;
        while (st < ie) {
          const int cc = split_owner(st, ap.W, p.G);
          const int en = min(ie, split_point(cc + 1, ap.W, p.G));
          const float ms = __ldcg(p.part_ml + (static_cast<size_t>(st) * GQ + h) * 2);
          const float lsg = __ldcg(p.part_ml + (static_cast<size_t>(st) * GQ + h) * 2 + 1);
          const float os = __ldcg(p.part_o + (static_cast<size_t>(st) * GQ + h) * D + dd);
          if (ms > M) {
            const float f = exp2f(M - ms);
            Ls = fmaf(Ls, f, lsg);
            Os = fmaf(Os, f, os);
            M = ms;
          } else if (ms != -INFINITY) {
            const float f = exp2f(ms - M);
            Ls = fmaf(lsg, f, Ls);
            Os = fmaf(os, f, Os);
          }
          st = en;
        }
        p.o[(static_cast<size_t>(seg_b) * p.nq + seg_g * GQ + h) * D + dd] = Os / Ls;
      }
      consumer_sync();
      if (cx.tid == 0) {
        atomicExch(arrive, 0u);
        release_add(p.cnt + l * ST_LAYER + ST_ATTN, 1u);
      }
    }
  }
}

// ------------------------------------------------------------------ stages

__device__ __forceinline__ const Mat& stage_mat(const LayerParams& L, int kind) {
  return kind == ST_QKV ? L.qkv : kind == ST_OPROJ ? L.o : kind == ST_GATEUP ? L.gu : L.down;
}

// Producer: the stream of one stage.
template <int D>
__device__ bool produce_stage(const Params& p, Ctx& cx, int kind, int l, int s, RingPos& rp,
                              uint64_t pol, bool fused) {
  const int where = where_code(kind, l, s) | (1 << 15);
  if (kind == ST_LM) return produce_gemv(p, cx, p.lm, rp, pol, where);
  if (kind == ST_ATTN) return produce_attn(p, cx, l, s, rp, pol, fused);
  const LayerParams& L = p.layers[l];
  return produce_gemv(p, cx, stage_mat(L, kind), rp, pol, where);
}

// Consumers: one stage.  Returns false once the CTA is aborting.
template <int B, int D>
__device__ bool consume_stage(const Params& p, Ctx& cx, int kind, int l, int s, RingPos& rp,
                              bool fused) {
  const unsigned G = static_cast<unsigned>(p.G);
  const unsigned S1 = static_cast<unsigned>(p.step_base + s + 1);
  const int where = where_code(kind, l, s);
  if (kind == ST_ATTN) {
    consume_attn<B, D>(p, cx, l, s, rp, fused);
    consumer_sync();
    return !cx.ctl->abort;
  }
  if (kind == ST_LM) {
    if (!stage_wait(p, cx, p.cnt + (p.L - 1) * ST_LAYER + ST_DOWN, G * S1, where, fused)) return false;
    float* hid = (p.hidden_out && cx.c == 0) ? p.hidden_out + static_cast<size_t>(s) * p.B * p.H : nullptr;
    load_act<B>(p, cx, p.H, SRC_RESID, p.x, p.final_norm, hid);
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    EpiLM<B> epi{p, s, &bv, &bi};
    consume_gemv<B>(p, cx, p.lm, rp, where, epi);
    if (cx.lane < B) {
      cx.ctl->red[cx.warp][cx.lane] = bv;
      cx.ctl->redi[cx.warp][cx.lane] = bi;
    }
    consumer_sync();
    if (cx.tid < B) {
      float v = -INFINITY;
      int ix = 0x7fffffff;
      for (int w = 0; w < kConsumerWarps; ++w) argmax_merge(v, ix, cx.ctl->red[w][cx.tid], cx.ctl->redi[w][cx.tid]);
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
        }
      }
      consumer_sync();
      if (cx.tid == 0) release_add(p.cnt + p.cl.step_done, 1u);
    }
    consumer_sync();
    return !cx.ctl->abort;
  }
  const LayerParams& L = p.layers[l];
  bool ok = true;
  switch (kind) {
    case ST_QKV: {
      if (l == 0) {
        ok = stage_wait(p, cx, p.cnt + p.cl.step_done, S1 - 1u, where, fused);
        if (!ok) return false;
        load_act<B>(p, cx, p.H, SRC_EMBED, nullptr, L.attn_norm, nullptr);
      } else {
        ok = stage_wait(p, cx, p.cnt + (l - 1) * ST_LAYER + ST_DOWN, G * S1, where, fused);
        if (!ok) return false;
        load_act<B>(p, cx, p.H, SRC_RESID, p.x, L.attn_norm, nullptr);
      }
      EpiQKV<B> epi{p, l, s};
      consume_gemv<B>(p, cx, L.qkv, rp, where, epi);
      break;
    }
    case ST_OPROJ: {
      const unsigned tgt = static_cast<unsigned>(p.B * p.nkv) * S1;
      if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_ATTN, tgt, where, fused)) return false;
      load_act<B>(p, cx, p.nq * p.d, SRC_PLAIN, p.o, nullptr, nullptr);
      EpiResid<B> epi{p, l == 0};
      consume_gemv<B>(p, cx, L.o, rp, where, epi);
      break;
    }
    case ST_GATEUP: {
      if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_OPROJ, G * S1, where, fused)) return false;
      load_act<B>(p, cx, p.H, SRC_RESID, p.x, L.ffn_norm, nullptr);
      EpiSwiGLU<B> epi{p};
      consume_gemv<B>(p, cx, L.gu, rp, where, epi);
      break;
    }
    default: {  // ST_DOWN
      if (!stage_wait(p, cx, p.cnt + l * ST_LAYER + ST_GATEUP, G * S1, where, fused)) return false;
      load_act<B>(p, cx, p.F, SRC_PLAIN, p.h, nullptr, nullptr);
      EpiResid<B> epi{p, false};
      consume_gemv<B>(p, cx, L.down, rp, where, epi);
      break;
    }
  }
  // KV entries written by the QKV epilogue are read by later steps through
  // the async proxy (bulk copies): order this thread's generic writes first.
  if (kind == ST_QKV) fence_proxy_async_global();
  consumer_sync();
  if (cx.tid == 0) release_add(p.cnt + l * ST_LAYER + kind, 1u);
  return !cx.ctl->abort;
}

// ------------------------------------------------------------------ kernels

__device__ __forceinline__ Ctx make_ctx(uint8_t* smem, const Params& p) {
  Ctx cx;
  cx.ring = smem;
  cx.act = reinterpret_cast<float*>(smem + static_cast<size_t>(p.nslot) * kSlotBytes);
  cx.ctl = reinterpret_cast<SmemCtl*>(smem + static_cast<size_t>(p.nslot) * kSlotBytes + p.act_bytes);
  cx.c = blockIdx.x;
  cx.tid = threadIdx.x;
  cx.warp = threadIdx.x >> 5;
  cx.lane = threadIdx.x & 31;
  return cx;
}

__device__ __forceinline__ void init_ring(const Params& p, Ctx& cx) {
  if (cx.tid == 0) {
    for (int i = 0; i < p.nslot; ++i) {
      mbar_init(smem_addr(&cx.ctl->full[i]), 1);
      mbar_init(smem_addr(&cx.ctl->empty[i]), kConsumerWarps);
    }
    cx.ctl->abort = 0;
    cx.ctl->flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
}

// Producer epilogue: wait until every issued copy has landed so the CTA's
// shared memory is not released under an in-flight bulk copy.
__device__ void drain_ring(const Params& p, Ctx& cx, const RingPos& rp, int issued) {
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
    const uint32_t fb = smem_addr(&cx.ctl->full[q.slot]);
    const uint64_t t0 = globaltimer();
    // Copies only read device memory and always complete; the bound (at least
    // 2 s, independent of the dependency-wait limit) only guards against a
    // device that stopped making progress.
    const long long limit = p.spin_limit_ns > 2000000000LL ? p.spin_limit_ns : 2000000000LL;
    while (!mbar_try_wait(fb, q.phase)) {
      if (static_cast<long long>(globaltimer() - t0) > limit) break;
    }
  }
}

template <int D>
__device__ void producer_main(const Params& p, Ctx& cx, int kind0, int l0, int s0, bool fused) {
  RingPos rp;
  const uint64_t pol = evict_first_policy();
  bool ok = true;
  if (fused) {
    for (int s = 0; s < p.n_steps && ok; ++s) {
      for (int l = 0; l < p.L && ok; ++l)
        for (int k = 0; k < ST_LAYER && ok; ++k) ok = produce_stage<D>(p, cx, k, l, s, rp, pol, true);
      if (ok) ok = produce_stage<D>(p, cx, ST_LM, 0, s, rp, pol, true);
    }
  } else {
    ok = produce_stage<D>(p, cx, kind0, l0, s0, rp, pol, false);
  }
  // Every slot's most recent copy must have landed before the CTA may exit.
  drain_ring(p, cx, rp, p.nslot);
}

template <int B, int D>
__device__ void consumer_main(const Params& p, Ctx& cx, int kind0, int l0, int s0, bool fused) {
  RingPos rp;
  if (fused) {
    for (int s = 0; s < p.n_steps; ++s) {
      for (int l = 0; l < p.L; ++l)
        for (int k = 0; k < ST_LAYER; ++k)
          if (!consume_stage<B, D>(p, cx, k, l, s, rp, true)) return;
      if (!consume_stage<B, D>(p, cx, ST_LM, 0, s, rp, true)) return;
    }
  } else {
    consume_stage<B, D>(p, cx, kind0, l0, s0, rp, false);
  }
}

// The persistent engine: one launch decodes p.n_steps tokens.
template <int B, int D>
__global__ void __launch_bounds__(kThreads, 1) engine_persistent(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctx cx = make_ctx(smem, p);
  init_ring(p, cx);
  if (cx.warp == kConsumerWarps) {
    if (cx.lane == 0) producer_main<D>(p, cx, 0, 0, 0, true);
    __syncwarp();
  } else {
    consumer_main<B, D>(p, cx, 0, 0, 0, true);
  }
}

// Kernel-per-op baseline: one launch runs one stage (same tiles, no waits).
template <int B, int D>
__global__ void __launch_bounds__(kThreads, 1) engine_stage(const __grid_constant__ Params p, int kind,
                                                            int layer, int step) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctx cx = make_ctx(smem, p);
  init_ring(p, cx);
  if (cx.warp == kConsumerWarps) {
    if (cx.lane == 0) producer_main<D>(p, cx, kind, layer, step, false);
    __syncwarp();
  } else {
    consumer_main<B, D>(p, cx, kind, layer, step, false);
  }
}

}  // namespace xlpk
