"""B200-native ReAttention top-k span attention (sm_100a CUDA behind a C ABI).

Import ``top_kv_span_b200.reatt`` for the binding; importing the package
itself loads nothing.
"""
