"""The bench's effective-FLOP numerator, checked on the CPU against pair counts
enumerated from the oracle's window definition: every query of a tile sees
the s keys of each tile in its kept list (sliding-tile branch), and every
query sees every pooled token (global branch), 4*d FLOP per pair forward."""
import pytest

import bench
from oracle import vattn_oracle as O
from synth import inputs as S


@pytest.mark.parametrize("name", ["tiny", "720p", "1080p", "4k", "train"])
def test_forward_flops_match_enumerated_pairs(name):
    w = S.WORKLOADS[name]
    g = O.geom_of(w)
    s = g.tile_volume
    kept = O.kept_tiles(g)
    pairs_local = w.batch * w.heads * sum(len(k) for k in kept) * s * s
    loc, glob = bench._flops_fwd(w)
    assert loc == 4 * w.head_dim * pairs_local
    if w.dual:
        assert glob == 4 * w.head_dim * w.batch * w.heads * g.n * g.n_pooled
    else:
        assert glob == 0


def test_720p_figure_of_the_bench_line():
    """1.4677e13 FLOP per 720p launch: 24 heads x 115200 queries x 27 tiles x 384 keys x 4 x 128."""
    loc, glob = bench._flops_fwd(S.WORKLOADS["720p"])
    assert glob == 0 and loc == 4 * 128 * 24 * 115200 * 27 * 384 == 14676708556800


def test_training_step_figures():
    """Training workload (B2, 1080p geometry): 7.368e13 FLOP forward and, at
    10*d per pair, 2.5 times that backward (1.842e14)."""
    loc, glob = bench._flops_fwd(S.WORKLOADS["train"])
    fwd = loc + glob
    assert round(fwd / 1e13, 3) == 7.368
    assert round(2.5 * fwd / 1e14, 3) == 1.842
