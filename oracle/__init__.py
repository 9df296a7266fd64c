"""CPU oracle for the NF4 grouped mixture-of-experts layer.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously
correct statement of what the GPU library computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  It shares no code, tables or constants
with the CUDA library and never imports it; the library never imports this.

Sources (web pages on the method, cited by page title and section):

* "Jordan Anderson" (jordananderson-pages.pages.dev), section
  "grouped-nf4-gemm & experts-4bit", first bullet: the MoE matmuls run on
  4-bit packed weights, one launch for all active experts, the codebook
  decoded inside the GEMM, the bitsandbytes packed layout consumed unchanged;
  third bullet: the codebook has sixteen entries (NF4).
* "Jordan Anderson" (jordananderson.work), section "4-bit Mixture-of-Experts
  fine-tuning on small GPUs", first two bullets: each MoE layer's experts are
  one fused 3-D parameter, and that fused stack is what gets quantized.
* The problem statement of this library fixes the rest: blocksize 64, fp32
  absmax, two codes per byte, top-k softmax routing, SiLU(gate)*up, a
  routing-weighted combine.
* The same pages mention GPTQ-calibrated int4 experts served by an INT4
  decode GEMV ("grouped-nf4-gemm & experts-4bit", third bullet; "MoE Training
  on Consumer GPUs", cerinamroth.com/ml, section "Task guides");
  ``oracle.int4`` states the format readings.
* Per-expert LoRA adapters over the frozen 4-bit base ("4-bit
  Mixture-of-Experts fine-tuning on small GPUs", jordananderson.work);
  ``oracle.lora`` states the readings.
* MXFP4 experts, e2m1 codes with an e8m0 scale per 32 ("grouped-nf4-gemm &
  experts-4bit", third bullet; "MoE Training on Consumer GPUs", "Task
  guides"); ``oracle.mxfp4`` states the readings.
* The layer's backward with the 4-bit experts frozen ("grouped-nf4-gemm &
  experts-4bit", jordananderson-pages.pages.dev, fourth bullet);
  ``oracle.backward`` states the readings.

Where the pages are silent the oracle takes one reading, documented at each
function.  Every function is pinned by tests in ``tests/test_oracle_*.py``
against closed forms, invariants, brute force and a published table; there
is no function whose parity is unpinned except the ones that say so.

Precision: decisions that produce integers (NF4 codes, top-k indices) are
taken in fp32, the precision the kernels use; everything else is fp64.
"""

from .nf4 import (  # noqa: F401
    BLOCKSIZE,
    nf4_levels,
    nf4_levels_from_quantiles,
    nf4_midpoints,
    quantize_blockwise,
    dequantize_blockwise,
    unpack_codes,
)
from .int4 import (  # noqa: F401
    GROUP as INT4_GROUP,
    quantize_int4_grouped,
    dequantize_int4_grouped,
    int4_scales_zeros,
)
from .mxfp4 import (  # noqa: F401
    BLOCK as MXFP4_BLOCK,
    e2m1_values,
    quantize_mxfp4,
    dequantize_mxfp4,
)
from .lora import lora_delta  # noqa: F401
from .backward import (  # noqa: F401
    grouped_gemm_t,
    swiglu_backward,
    combine_backward,
    route_backward,
    moe_layer_backward,
    moe_layer_backward_permuted,
    lora_backward,
)
from .routing import route_topk, permute_by_expert  # noqa: F401
from .moe import (  # noqa: F401
    swiglu,
    grouped_gemm,
    grouped_gemm_int4,
    grouped_gemm_mxfp4,
    unpermute_combine,
    moe_layer,
    moe_layer_dense,
    moe_layer_permuted,
    ExpertStack,
    Int4ExpertStack,
    Mxfp4ExpertStack,
)
