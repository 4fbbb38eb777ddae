"""fp64 CPU oracle for dual-branch (sliding-tile local + pooled global) 3D attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product library imports, links or
runs this package; only the test suite, the smoke check and the benchmark's
CPU-baseline leg use it.  It shares no code with the CUDA path.

Every function is a plain restatement of the definitions in:
  * "UltraGen: High-Resolution Video Generation with Hierarchical Attention"
    §3 (token grid, full attention), §4.1 (global-local decomposition and the
    fusion factor), §4.2 (spatially compressed global attention),
    App. B (complexity);
  * "Fast Video Generation with Sliding Tile Attention", abstract (tile-by-tile
    sliding 3D windows);
  * "AtlasVid: Efficient Ultra-High-Resolution Long Video Generation via
    Decoupled Global-Local Modeling", abstract (reordered spatiotemporal
    windows, asymmetric global-local attention: only K/V are compressed).
"""
from .vattn_oracle import *  # noqa: F401,F403
