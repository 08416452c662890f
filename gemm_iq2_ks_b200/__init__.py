"""B200-native (sm_100a) IQ2_KS / IQ2_K routed-expert kernels.

The product is the C-ABI library ``libiqk.so`` (include/iqk.h); this package
builds it in-tree (``build.py``) and exposes a thin ctypes binding with the
same entry-point names (``gemm_iq2_ks_b200.binding``). Importing the package
does not load the library; the first call through the binding does.
"""
