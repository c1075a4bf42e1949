// dq_solve_qch.cu — the solve kernel instantiated with the Q-change trace (Figure 2 (a) of
// the DualQuant paper); compiled apart from the plain instantiations so the two build in
// parallel.
#include "dq_solve_kernel.cuh"

namespace dq {

cudaError_t launch_solve_qch(const SolveLaunch& L, int count, int kind, int group, int esize,
                             const SolvePlan& p, cudaStream_t s) {
  return launch_solve_formats<true>(L, count, kind, group, esize, p, s);
}

}  // namespace dq
