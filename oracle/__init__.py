"""Float64 CPU oracle (test infrastructure only; never imported by the library)."""
from .gdn_ref import default_key_scale, gdn_scan_ref, rel_frobenius

__all__ = ["default_key_scale", "gdn_scan_ref", "rel_frobenius"]
