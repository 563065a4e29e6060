"""B200-native (sm_100a) Gated DeltaNet token mixer: prefill and decode through a C ABI.

    from gated_deltanet_token_b200 import gdn
    y, final_state = gdn.gdn_prefill(q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, ...)
"""
__all__ = ["gdn", "inputs"]
