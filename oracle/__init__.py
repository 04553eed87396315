"""CPU oracle for SageAttention-style quantized attention.

TEST INFRASTRUCTURE, not product code.  Only the test-suite, the smoke
check of the package entry file and the benchmark's CPU-baseline /
reference legs may import it.  The CUDA path never imports, links or calls
anything in here, and this package never imports the CUDA path: the two
share only the seeded input generator (``workloads``), which holds none of
the method's arithmetic.
"""
from .codecs import e4m3_decode, e4m3_encode, e4m3_round, fp16_rne, E4M3_MAX, FP16_MAX
from .sage import (BLOCK, rope, mean_k, quant_blocks, quant_q, smooth_quant_k, quant_v_fp8,
                   attention_reference, attention_online, sage_attention, sage_attention_varlen,
                   f16acc_product_limit, f16acc_bound_ok, cossim, rel_l1, rmse)
