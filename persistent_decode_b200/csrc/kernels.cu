// One compilation unit of decode-kernel instantiations: built with
// -DXLPK_UNIT=n for n in [0, kKernelUnits), each unit the variants its
// XLPK_UNITn list names.
#include "engine.cuh"
#include "kernels.h"

#ifndef XLPK_UNIT
#error "XLPK_UNIT selects the instantiations of this unit"
#endif

namespace xlpk {

template <int B, int D, bool MOE, int VAR>
void launch_stage_impl(const Params& p, int kind, int layer, int step, int grid, int smem, cudaStream_t st) {
  engine_stage<B, D, MOE, VAR><<<grid, kThreads, smem, st>>>(p, kind, layer, step);
}

template <int B, int D, bool MOE, int VAR>
KernelSet kernel_set() {
  return KernelSet{reinterpret_cast<const void*>(&engine_persistent<B, D, MOE, VAR>),
                   reinterpret_cast<const void*>(&engine_stage<B, D, MOE, VAR>),
                   &launch_stage_impl<B, D, MOE, VAR>};
}

#define XLPK_INST_SET(b, d, m, k) template KernelSet kernel_set<b, d, m, k>();
#if XLPK_UNIT == 0
XLPK_UNIT0(XLPK_INST_SET)
#elif XLPK_UNIT == 1
XLPK_UNIT1(XLPK_INST_SET)
#elif XLPK_UNIT == 2
XLPK_UNIT2(XLPK_INST_SET)
#elif XLPK_UNIT == 3
XLPK_UNIT3(XLPK_INST_SET)
#elif XLPK_UNIT == 4
XLPK_UNIT4(XLPK_INST_SET)
#elif XLPK_UNIT == 5
XLPK_UNIT5(XLPK_INST_SET)
#elif XLPK_UNIT == 6
XLPK_UNIT6(XLPK_INST_SET)
#elif XLPK_UNIT == 7
XLPK_UNIT7(XLPK_INST_SET)
#elif XLPK_UNIT == 8
XLPK_UNIT8(XLPK_INST_SET)
#elif XLPK_UNIT == 9
XLPK_UNIT9(XLPK_INST_SET)
#elif XLPK_UNIT == 10
XLPK_UNIT10(XLPK_INST_SET)
#else
#error "XLPK_UNIT out of range"
#endif
#undef XLPK_INST_SET

}  // namespace xlpk
