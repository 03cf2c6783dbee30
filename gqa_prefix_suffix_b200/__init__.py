"""B200 (sm_100a) suffix attention of the DM0.5 action expert.

The work is done by the CUDA library ``libdm05_suffix_attn.so`` (C ABI in
``include/dm05_suffix_attn.h``); ``binding`` marshals arguments to it.
"""
from .binding import (Dm05Error, dm05_get_error_word, dm05_release, dm05_set_split_override,  # noqa: F401
                      dm05_status_string, dm05_suffix_attn, dm05_suffix_attn_plan,
                      dm05_suffix_attn_reserve, dm05_suffix_attn_workspace_bytes, reserve_for,
                      suffix_attn)
