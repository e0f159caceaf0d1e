"""Plain fp64 CPU oracle for the dynamic block-sparse attention path.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.
"""
from .sparse_attn_ref import *  # noqa: F401,F403
from .sparse_attn_ref import (BLOCK, E4M3_MAX, attn_int8fp8_from_codes, attn_ref_exact,  # noqa: F401
                              attn_ref_int8fp8, block_means, block_scores, e4m3_decode,
                              e4m3_encode, e4m3_round, keep_count, kth_threshold, max_abs_err,
                              n_blocks, plan_mask, plan_ref, quant_qk_ref, quant_v_ref,
                              rel_l1_err, select_topk)
from .prologue_ref import (ROPE_THETA, bf16_round, k_channel_mean_ref, prologue_ref,  # noqa: F401
                           qk_rmsnorm_ref, quant_k_smooth_ref, rope3d_ref, rope3d_split, token_positions)
from .ulysses_ref import (all_to_all_ref, fp8_rows_dequant_ref, fp8_rows_ref, pack_o_ref, pack_qkv_ref,  # noqa: F401
                          unpack_o_ref, unpack_qkv_ref)
from .nvfp4_ref import (E2M1_MAX, NVFP4_BLOCK, dequant_nvfp4_ref, e2m1_decode, e2m1_encode,  # noqa: F401
                         e2m1_round, gemm_nvfp4_ref, nvfp4_global_scale, pack_e2m1, quant_nvfp4_ref, sf_tiled,
                         unpack_e2m1)
