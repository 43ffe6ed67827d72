"""Float64 CPU oracles (test infrastructure only; never imported by the library)."""
from .conv_ref import temporal_conv_ref
from .gdn_ref import default_key_scale, gdn_scan_ref, rel_frobenius

__all__ = ["default_key_scale", "gdn_scan_ref", "rel_frobenius", "temporal_conv_ref"]
