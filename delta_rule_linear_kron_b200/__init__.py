"""Kronecker delta rule (KronLSTM token mixer) for NVIDIA B200 (sm_100a)."""
