"""Pins of the oracle's accounting to the figures the pages print (CPU).
Each fixture under tests/golden/ carries its source in its header."""
import os

from oracle import vattn_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, val = (x.strip() for x in line.split("="))
                vals[key] = int(val)
    return vals


def test_attention_map_grows_sixteenfold_when_height_and_width_double():
    """Full attention = the local branch with a window covering the grid;
    its pair count, and the brute-force token mask, both grow by the printed
    factor."""
    gold = _load("ultragen_s3_attention_map_scaling.txt")
    for (T, H, W), tile in [((4, 8, 8), (2, 4, 4)), ((21, 72, 120), (3, 8, 8)), ((30, 48, 80), (6, 8, 8))]:
        def full(h, w):
            g = O.Geom(T, h, w, tile, (1, 1, 1))
            return g._replace(window=g.tiles_per_dim)
        g1, g2 = full(H, W), full(2 * H, 2 * W)
        assert g2.n == gold["token_ratio"] * g1.n
        assert O.kept_pairs_local(g2, 1, 1) == gold["attention_map_ratio"] * O.kept_pairs_local(g1, 1, 1)
        assert O.kept_pairs_local(g1, 1, 1) == g1.n ** 2
    # the brute-force mask on a tiny grid: every token pair, sixteen times as many
    g1 = O.Geom(2, 4, 4, (1, 2, 2), (2, 2, 2))
    g2 = O.Geom(2, 8, 8, (1, 2, 2), (2, 4, 4))
    assert O.sta_mask_bruteforce(g2).sum() == gold["attention_map_ratio"] * O.sta_mask_bruteforce(g1).sum()


def test_appendix_b_speedup_at_k4():
    gold = _load("ultragen_appB_speedup.txt")
    assert round(1 / O.ultragen_cost_ratio(gold["K"])) == gold["approx_speedup"]


def test_fixtures_cite_their_source():
    for name in os.listdir(GOLDEN):
        head = open(os.path.join(GOLDEN, name)).read()
        assert head.startswith("# Source: "), name
