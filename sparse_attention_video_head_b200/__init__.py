"""SVG2 semantic-aware permuted sparse attention for one DiT attention layer, native on B200.

The product is the C-ABI library libsvg2.so (include/svg2.h, sources in csrc/); the `svg2`
module is its Python binding and `inputs` draws the seeded synthetic layer inputs.  Importing
the package loads nothing; `sparse_attention_video_head_b200.svg2.lib()` loads the library and
raises if it has not been built.
"""
__all__ = ["svg2", "inputs", "build"]
