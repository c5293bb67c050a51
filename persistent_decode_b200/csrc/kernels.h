// Instantiations of the decode kernels, compiled in separate translation units
// (kernels.cu built once per unit below) so the build runs them in parallel.
// The host side reaches a variant only through its KernelSet.
#pragma once

#include <cuda_runtime.h>

#include "params.h"

namespace xlpk {

struct KernelSet {
  const void* persistent;   // engine_persistent<B, D, MOE, VAR>
  const void* stage;        // engine_stage<B, D, MOE, VAR>
  void (*launch_stage)(const Params& p, int kind, int layer, int step, int grid, int smem, cudaStream_t st);
};

// B sequences, head_dim D, MoE FFN, VAR: bit 0 an e4m3 KV cache, bit 1 NVFP4 weights.
template <int B, int D, bool MOE, int VAR>
KernelSet kernel_set();

// Every built variant, grouped by compilation unit (XLPK_UNIT = 0..10).
#define XLPK_UNIT0(X) X(1, 64, false, 0) X(1, 128, false, 0)
#define XLPK_UNIT1(X) X(1, 64, true, 0) X(1, 128, true, 0)
#define XLPK_UNIT2(X) X(1, 64, false, 1) X(1, 128, false, 1)
#define XLPK_UNIT3(X) X(2, 64, false, 0) X(2, 128, false, 0)
#define XLPK_UNIT4(X) X(2, 64, false, 1) X(2, 128, false, 1)
#define XLPK_UNIT5(X) X(4, 64, false, 0) X(4, 128, false, 0)
#define XLPK_UNIT6(X) X(4, 64, false, 1) X(4, 128, false, 1)
#define XLPK_UNIT7(X) X(8, 64, false, 0) X(8, 128, false, 0)
#define XLPK_UNIT8(X) X(8, 64, false, 1) X(8, 128, false, 1)
#define XLPK_UNIT9(X) X(1, 64, false, 2) X(1, 128, false, 2)
#define XLPK_UNIT10(X) X(1, 64, false, 3) X(1, 128, false, 3)
constexpr int kKernelUnits = 11;

#define XLPK_EXTERN_SET(b, d, m, k) extern template KernelSet kernel_set<b, d, m, k>();
XLPK_UNIT0(XLPK_EXTERN_SET)
XLPK_UNIT1(XLPK_EXTERN_SET)
XLPK_UNIT2(XLPK_EXTERN_SET)
XLPK_UNIT3(XLPK_EXTERN_SET)
XLPK_UNIT4(XLPK_EXTERN_SET)
XLPK_UNIT5(XLPK_EXTERN_SET)
XLPK_UNIT6(XLPK_EXTERN_SET)
XLPK_UNIT7(XLPK_EXTERN_SET)
XLPK_UNIT8(XLPK_EXTERN_SET)
XLPK_UNIT9(XLPK_EXTERN_SET)
XLPK_UNIT10(XLPK_EXTERN_SET)
#undef XLPK_EXTERN_SET

}  // namespace xlpk
