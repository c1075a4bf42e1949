// dq_solve_int8.cu — the solve kernel instantiated for the 8-bit formats INT8 (G=128 or 64,
// bf16 block scales) and MXINT8 (G=32, E8M0): the DualQuant appendix's 8-bit table and the
// acceptodds abstract's format list. Same solver with q_max = 127 and one code byte per
// element; compiled apart (the extended instantiation in dq_solve_int8_ext.cu) so the
// translation units build in parallel.
#include "dq_solve_kernel.cuh"

namespace dq {

cudaError_t launch_solve_8bit(const SolveLaunch& L, int count, int kind, int group, int esize,
                              const SolvePlan& p, bool ext, cudaStream_t s) {
  if (ext) return launch_solve_8bit_ext(L, count, kind, group, esize, p, s);
  return launch_solve_formats8<false>(L, count, kind, group, esize, p, s);
}

}  // namespace dq
