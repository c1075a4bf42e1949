"""Plain CPU oracle of the DualQuant hot path (TEST INFRASTRUCTURE ONLY).

A slow, obviously-correct NumPy restatement of the dual-scale BCD weight-reconstruction
solver and of the activation rescale + 4-bit quantization, written from the DualQuant pages:

  * "DualQuant: Dual-scale Calibration-free Weight-and-Activation Quantization for LLMs"
    (thelatestinai.com/papers/2610.13767), Abstract, Figures 1-3, appendix Table 6;
  * the same paper's abstract on acceptodds.com/papers/iclr2027-49818 (black-box quantizer,
    projection of the scales onto the format's admissible set after every update);
  * the ai4snews.wisdomeyes.cn summary (one row scale and one column scale per matrix;
    the column scales act as activation rescalings).

Floating point is binary64 throughout, except where a binary32 value decides an integer
(an element code or a scale code): there both this oracle and the CUDA path take the
decision on the same binary32 value (see `formats` and `solver.q_step`).

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline leg may import this
package. It shares no code with the CUDA path and imports nothing from it.

Pins: every public function is checked by `tests/test_oracle_*.py` against library
conversions (torch float8/bfloat16), brute force on tiny inputs, closed forms and
invariants. Parity unpinned: the pages print no worked numeric example, so the 12.54x
MSE ratio of Figure 1 and the SQNR values of Table 6 cannot be reproduced.
"""
from .formats import Format, FORMAT_KINDS, make_format  # noqa: F401
from .solver import solve, q_step, r_step, c_step, mse, init_scales  # noqa: F401
from .actquant import act_quant, sqnr  # noqa: F401
