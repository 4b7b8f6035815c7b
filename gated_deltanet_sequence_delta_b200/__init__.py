"""Gated DeltaNet core (gated delta rule) for NVIDIA B200, sm_100a.

The computation lives in ``libgdn.so`` (C ABI: ``include/gdn.h``); this package
is its thin binding.  Names are re-exported lazily so that ``inputs`` (the
seeded workload generator) can be imported without loading torch or the
library.
"""
_BINDING = ("gdn_gates", "gdn_chunk_prefill", "gdn_chunk_prefill_gated", "gdn_chunk_prefill_outgate", "gdn_chunk_prefill_status",
            "gdn_conv_prefill", "gdn_conv_status", "gdn_cp_segment", "gdn_cp_combine", "gdn_cp_status", "gdn_decode_step", "gdn_decode_step_gated", "gdn_decode_step_fused",
            "gdn_decode_status", "gdn_chunk_prefill_host", "prefill_host_workspace_bytes",
            "GDNError", "GDNLibraryError", "prefill_workspace_bytes", "kernel_launches", "testing_stall",
            "STALL_NONE", "STALL_DECODE", "STALL_PREFILL_PREP")

__all__ = list(_BINDING)


def __getattr__(name):
    if name in _BINDING:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
