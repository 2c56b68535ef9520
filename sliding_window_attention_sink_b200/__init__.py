"""B200-native sliding-window / global causal GQA attention with a per-head
attention sink (MiMo Hybrid SWA), behind a C-ABI library ``libswasink.so``.

Import is cheap: the CUDA library is loaded on first use by
:mod:`sliding_window_attention_sink_b200.binding`, which raises if it is
missing. There is no CPU fallback.
"""
__all__ = ["binding", "workloads"]
