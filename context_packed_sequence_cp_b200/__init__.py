"""thdcp: packed-sequence (THD) causal attention with EOD resets under load-balanced
KV-all-gather context parallelism, as a C-ABI CUDA library for B200 (sm_100a) with a
thin Python binding.  All context-parallel ranks are virtual ranks on one GPU.

Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance".
"""
from .api import (Plan, thd_cp_attn_bwd, thd_cp_attn_bwd_noalloc, thd_cp_attn_bwd_workspace,  # noqa: F401
                  thd_cp_attn_fwd, thd_cp_attn_fwd_fused_gather, thd_cp_attn_fwd_mla, thd_cp_plan,
                  thd_cu_seqlens_from_eod, thd_kv_gather,
                  thd_position_ids, thd_rope_apply, thd_rows_to_global)
from ._lib import ThdError, lib  # noqa: F401
