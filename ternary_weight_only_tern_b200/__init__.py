"""B200-native weight-only ternary linear layer (W1.58A16): packing, the decode GEMV and
prefill GEMM on packed planes, and bit accounting, behind the C-ABI library libtern.so.

    from ternary_weight_only_tern_b200 import TernWeight, linear, pack_exec, bits

The torch front end (api) is imported on first use, so that ``synth`` (seeded inputs)
imports without PyTorch or the library.
"""

_API = ("TernWeight", "linear", "workspace_bytes", "pack_exec", "unpack_exec", "pack_store",
        "unpack_store", "weight_validate", "bits")


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)


__all__ = list(_API)
