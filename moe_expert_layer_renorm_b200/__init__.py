"""NVFP4 MoE FFN layer for B200 (sm_100a): C-ABI library + thin Python binding."""
