"""B200-native Mamba hot path: causal conv1d, fused prefill selective scan and
single-token selective_state_update, behind the C-ABI library
``libssm_causal.so`` (declared in ``include/ssm_causal.h``)."""
