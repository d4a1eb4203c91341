"""CPU oracle for the MXFP4 MoE block-verify path -- TEST INFRASTRUCTURE.

Plain, slow, obviously-correct numpy code in float64 that states what the
path computes.  It is the yardstick the CUDA library is checked against and
it is never on the product path: only the test-suite, the package smoke check
and the benchmark's CPU-baseline leg may import it.  It shares no code with
the CUDA library (no kernels, headers, tables or helpers); the two meet only
in the seeded input generator, which holds none of the method's arithmetic.

Modules
  mxfp4   -- OCP MXFP4 decoding (E2M1 element codes, E8M0 block scales),
             an encoder used for round-trip checks, bf16 rounding.
  moe     -- top-k routing, permutation by expert, SwiGLU expert FFN over
             dequantised weights, weighted combine, the parameter-free
             RMSNorm between stacked layers.
  accept  -- greedy prefix acceptance and speculative rejection sampling.

Sources, cited by page title and section:
  [P1] "mimo-v2-5-speculative-decoding-draft-scheduling" (blog.hotdry.top)
  [P2] "如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？" (zhihu answer)
  [P3] "MiMo-v2.5-Pro-UltraSpeed - infra 架构解读" (hotpursuit.aufer.space)
  [P4] "mimo-tilert-1000tps-trillion-parameter-inference" (blog.hypho.cn)
  [OCP] OCP Microscaling Formats (MX) Specification v1.0, the format that
        [P3] section "FP4 Expert 量化" and [P4] section "第一层：FP4 选择性量化"
        name for the expert weights.

Parity status: every function here is pinned by `-m "not gpu"` tests against
values fixed outside this package (OCP value table, closed forms, brute force,
library routines, a chi-square test of losslessness).  No function is
"parity unpinned".
"""
from . import mxfp4, moe, accept  # noqa: F401
