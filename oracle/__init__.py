"""CPU oracle for the fused exact-attention forward pass (test infrastructure).

This package is test infrastructure, not product code.  Only the tests, the
package smoke check and the CPU-baseline / reference arm of ``bench.py`` may
import it.  The CUDA path never imports it, and it imports nothing from the
CUDA path: the two share no code, constants or helpers.

Sources cited in this package (web pages on FlashAttention):

* [AY]  AllenY's blog, "FlashAttention" post (alleny.xyz/post/flashattention):
        sections "(Safe) Softmax", "从3-pass到2-pass", "FlashAttention".
* [WM]  wmrh.cn article on FlashAttention (news/298785): sections
        "2.1 Online Softmax", "2.2 把 Online Softmax 嵌入注意力".
* [UF]  "理解 Flash Attention：在 Triton 中从头编写算法" (Understanding Flash
        Attention: writing it from scratch in Triton): sections "什么是注意力",
        "瓦片注意力计算", "算法概述".

Modules:

* ``softmax``        -- 3-pass safe softmax, 2-pass online softmax, and the
                        concatenated-softmax merge rule.
* ``attention``      -- the definition of masked scaled-dot-product attention
                        and its logsumexp in float64 (NumPy), plus the one-pass
                        tiled algorithm written in the pages' order.
* ``brute``          -- an independent pure-Python version for tiny shapes.
* ``backward``       -- dQ, dK, dV by the chain rule through the definition.
* ``varlen``         -- variable-length batches: independent sequences packed
                        token-major without padding.
* ``fp8``            -- the E4M3 format written out, attention of the real
                        values 8-bit codes stand for, and the weighted spread
                        of V that bounds the effect of rounding P.

Every function here is pinned by ``tests/test_oracle.py`` to closed forms,
invariants and the pages' worked example; see that file's header.
"""

from .softmax import safe_softmax_3pass, online_softmax_2pass, merge_partials  # noqa: F401
from .attention import (  # noqa: F401
    visible_mask,
    attention_ref,
    attention_ref_rows,
    attention_tiled_online,
)
from .brute import attention_brute  # noqa: F401
from .backward import attention_bwd_ref, softmax_delta  # noqa: F401
from .varlen import attention_varlen_ref  # noqa: F401
from .fp8 import attention_fp8_ref, e4m3_decode, weighted_spread  # noqa: F401
