// dq_solve_ext.cu — the extended instantiation of the solve kernel: the row-only and
// column-only update modes (the ablation of the ai4snews summary of DualQuant, paragraph 2)
// and the Q-change trace (Figure 2 (a) of the DualQuant paper). Kept apart from the plain
// instantiation, which therefore carries none of their flags, and compiled in parallel.
#include "dq_solve_kernel.cuh"

namespace dq {

cudaError_t launch_solve_ext(const SolveLaunch& L, int count, int kind, int group, int esize,
                             const SolvePlan& p, cudaStream_t s) {
  return launch_solve_formats<true>(L, count, kind, group, esize, p, s);
}

}  // namespace dq
