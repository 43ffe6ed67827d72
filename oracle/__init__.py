"""Float64 CPU oracles (test infrastructure only; never imported by the library)."""
from .conv_ref import temporal_conv_ref
from .gdn_ref import default_key_scale, gdn_scan_ref, rel_frobenius
from .rope_ref import rope3d_ref, rope_angles, rope_sections

__all__ = ["default_key_scale", "gdn_scan_ref", "rel_frobenius", "temporal_conv_ref",
           "rope3d_ref", "rope_angles", "rope_sections"]
