"""GPTQ-family per-layer solve on B200 (sm_100a): thin binding over libgptq.so."""
