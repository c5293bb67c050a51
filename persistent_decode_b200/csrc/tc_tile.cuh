// Tensor-core GEMM tile for the batch-8 projections (5th-generation tensor
// cores: tcgen05.mma with the accumulator in tensor memory).
//
// At batch 8 each weight element of a projection meets 8 activations, so the
// GEMV becomes a dense contraction Y[N][8] = W[N][K] . X[8][K]^T that the
// CUDA-core path would have to run at 16 flop per weight byte.  Here one CTA
// owns 128 rows of W: the elected thread streams W in [128 rows][64 columns]
// boxes with a 2-D TMA copy (128-byte swizzle), and issues
// tcgen05.mma.cta_group::1.kind::f16 with A = the weight box (M = 128,
// K-major) and B = the CTA's activations (N = 16: the 8 sequences plus 8 zero
// rows, bf16, K-major, same swizzle), accumulating fp32 in 16 tensor-memory
// columns.  The four warps then read their 32 rows of the accumulator
// (tcgen05.ld 32x32b) and store them.
//
// Operand layouts follow the canonical K-major SWIZZLE_128B form of the
// tcgen05 shared-memory matrix descriptor: rows of 128 bytes (64 bf16), the
// 16-byte chunks of row r XOR-permuted by r mod 8, 8-row groups 1024 bytes
// apart; a K step of 16 elements advances the descriptor's start address by
// 32 bytes inside the swizzle atom.
//
// Every wait is bounded: a wait that runs out records XLPK_ERR_TIMEOUT in
// *err, waits (bounded again) for the copy or the MMAs still in flight, frees
// the tensor memory and leaves.
#pragma once
#include "engine.cuh"
#include "tcgen05.cuh"

namespace xlpk {

constexpr int kTcRows = 128;       // M: weight rows per CTA
constexpr int kTcN = 16;           // N: 8 sequences + 8 zero rows
constexpr int kTcKBox = 64;        // columns per TMA box (128 bytes of bf16)
constexpr int kTcMaxK = 4096;      // activations of all K stay in shared memory
constexpr int kTcThreads = 128;    // 4 warps: one per 32-lane tensor-memory sub-partition
constexpr int kTcTmemCols = 32;    // allocation granularity (>= kTcN fp32 columns)

__host__ __device__ constexpr int tc_smem_bytes(int K) {
  return 1024 /* alignment slack */ + kTcRows * 128 /* A box */ + (K / kTcKBox) * kTcN * 128 /* B */ + 64;
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = kTcN, M = kTcRows.
constexpr uint32_t kTcIdesc = tc_idesc_bf16(kTcRows, kTcN);

// Bounded wait on an mbarrier phase (plain polling; the tile is short).
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, long long limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (static_cast<long long>(globaltimer() - t0) > limit_ns) return false;
  }
  return true;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_tile_kernel(const __grid_constant__ CUtensorMap wmap, int N, int K, const float* __restrict__ x,
                        float* __restrict__ y, int* err, long long limit_ns) {
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  const int nk = K / kTcKBox;
  uint8_t* a_box = base;                              // [128 rows][64] bf16, swizzled
  uint8_t* b_ops = base + kTcRows * 128;              // nk x [16 rows][64] bf16, swizzled
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_ops + nk * kTcN * 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  int* ok_flag = reinterpret_cast<int*>(bars + 3);
  const uint32_t full = smem_addr(&bars[0]), mma_done = smem_addr(&bars[1]);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * kTcRows;

  // Activations -> bf16 B operand, rows 0..7 the sequences, rows 8..15 zero.
  for (int u = tid; u < nk * kTcN * 8; u += kTcThreads) {
    const int kc = u / (kTcN * 8), rem = u - kc * (kTcN * 8);
    const int r = rem >> 3, ch = rem & 7;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (r < 8) {
      const float4* src = reinterpret_cast<const float4*>(x + static_cast<size_t>(r) * K + kc * kTcKBox + ch * 8);
      const float4 lo = __ldg(src), hi = __ldg(src + 1);
      w[0] = pack_bf16x2(lo.x, lo.y);
      w[1] = pack_bf16x2(lo.z, lo.w);
      w[2] = pack_bf16x2(hi.x, hi.y);
      w[3] = pack_bf16x2(hi.z, hi.w);
    }
    const uint32_t dst = smem_addr(b_ops) + kc * (kTcN * 128) + r * 128 + (((ch ^ (r & 7))) << 4);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3])
                 : "memory");
  }
  // the MMAs read the operand through the async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(mma_done, 1);
    *ok_flag = 1;
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (tid == 0) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    const uint32_t a_s = smem_addr(a_box), b_s = smem_addr(b_ops);
    bool ok = true;
    for (int kc = 0; kc < nk && ok; ++kc) {
      mbar_expect_tx(full, kTcRows * 128);
      tma_load_2d(a_s, &wmap, kc * kTcKBox, row0, full, pol);
      if (!tc_wait(full, kc & 1, limit_ns)) {
        ok = false;
        tc_wait(full, kc & 1, 4 * limit_ns);   // the copy still owns the box
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kTcKBox / 16; ++ks)
        tc_mma(tmem, tc_desc_sw128(a_s + ks * 32), tc_desc_sw128(b_s + kc * (kTcN * 128) + ks * 32), kTcIdesc,
               (kc | ks) != 0 ? 1u : 0u);
      // the next box overwrites A: wait until these MMAs have read it
      tc_commit(mma_done);
      if (!tc_wait(mma_done, kc & 1, limit_ns)) {
        ok = false;
        tc_wait(mma_done, kc & 1, 4 * limit_ns);
      }
    }
    if (!ok) {
      *ok_flag = 0;
      atomicExch(err, static_cast<int>(kErrTimeout));
    }
  }
  __syncthreads();
  tc_fence_after();
  if (*reinterpret_cast<volatile int*>(ok_flag)) {
    // warp w reads accumulator rows 32w .. 32w+31 (its tensor-memory lanes),
    // columns 0..7 (the sequences)
    uint32_t v[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
        : "r"(tmem + (static_cast<uint32_t>(warp * 32) << 16)));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    const int row = row0 + warp * 32 + lane;
    if (row < N) {
      float4* dst = reinterpret_cast<float4*>(y + static_cast<size_t>(row) * 8);
      dst[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]), __uint_as_float(v[3]));
      dst[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]), __uint_as_float(v[7]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols)
                 : "memory");
  }
}

}  // namespace xlpk
