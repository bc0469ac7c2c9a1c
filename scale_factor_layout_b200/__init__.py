"""scale_factor_layout_b200: MXFP8 E8M0 scale factors -> per-group 128x4 blocked layout on B200."""
