// Instantiations of the decode kernels, compiled in separate translation units
// (kernels.cu built once per unit below) so the build runs them in parallel.
// The host side reaches a variant only through its KernelSet.
#pragma once

#include <cuda_runtime.h>

#include "params.h"

namespace xlpk {

struct KernelSet {
  const void* persistent;   // engine_persistent<B, D, MOE, KV8>
  const void* stage;        // engine_stage<B, D, MOE, KV8>
  void (*launch_stage)(const Params& p, int kind, int layer, int step, int grid, int smem, cudaStream_t st);
};

// B sequences, head_dim D, MoE FFN, e4m3 KV cache.
template <int B, int D, bool MOE, bool KV8>
KernelSet kernel_set();

// Every built variant, grouped by compilation unit (XLPK_UNIT = 0..8).
#define XLPK_UNIT0(X) X(1, 64, false, false) X(1, 128, false, false)
#define XLPK_UNIT1(X) X(1, 64, true, false) X(1, 128, true, false)
#define XLPK_UNIT2(X) X(1, 64, false, true) X(1, 128, false, true)
#define XLPK_UNIT3(X) X(2, 64, false, false) X(2, 128, false, false)
#define XLPK_UNIT4(X) X(2, 64, false, true) X(2, 128, false, true)
#define XLPK_UNIT5(X) X(4, 64, false, false) X(4, 128, false, false)
#define XLPK_UNIT6(X) X(4, 64, false, true) X(4, 128, false, true)
#define XLPK_UNIT7(X) X(8, 64, false, false) X(8, 128, false, false)
#define XLPK_UNIT8(X) X(8, 64, false, true) X(8, 128, false, true)
constexpr int kKernelUnits = 9;

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
#undef XLPK_EXTERN_SET

}  // namespace xlpk
