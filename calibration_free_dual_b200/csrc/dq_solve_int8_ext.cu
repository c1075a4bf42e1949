// dq_solve_int8_ext.cu — the extended instantiation (update modes, Q-change trace) of the
// solve kernel for the 8-bit formats INT8 and MXINT8.
#include "dq_solve_kernel.cuh"

namespace dq {

cudaError_t launch_solve_8bit_ext(const SolveLaunch& L, int count, int kind, int group,
                                  int esize, const SolvePlan& p, cudaStream_t s) {
  return launch_solve_formats8<true>(L, count, kind, group, esize, p, s);
}

}  // namespace dq
