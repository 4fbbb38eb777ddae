"""The ctypes binding marshals arguments only (CPU; the library is replaced
by a recording fake, so nothing is launched): every wrapper passes as many
arguments as the C signature declares, and tensor arguments are checked for
contiguity and for the side (device or host) the C argument lives on."""
import pytest
import torch


class FakeTensor:
    """Stands in for a CUDA tensor on a machine without one."""

    def __init__(self, addr=4096, cuda=True, contiguous=True, shape=(1, 2, 256, 64), elem=2):
        self.addr, self.is_cuda, self._contig, self.shape, self.elem = addr, cuda, contiguous, shape, elem

    def data_ptr(self):
        return self.addr

    def is_contiguous(self):
        return self._contig

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        return self.elem

    def dim(self):
        return len(self.shape)


class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def B(monkeypatch):
    import video_dit_local_b200.binding as B
    fake = FakeLib()
    monkeypatch.setattr(B, "lib", fake)
    monkeypatch.setattr(B, "_stream", lambda s: None)
    B.fake = fake
    yield B
    del B.fake


def _geom(B):
    return B.make_geom(1, 2, 64, (4, 8, 8), (2, 4, 4), (1, 2, 2), (1, 2, 2))


def _calls(B):
    t = FakeTensor
    g = _geom(B)
    h = dict(cuda=False)
    return {
        "vattn_tile_permute": lambda: B.vattn_tile_permute(g, t(), t()),
        "vattn_tile_unpermute": lambda: B.vattn_tile_unpermute(g, t(), t()),
        "vattn_kept_tiles": lambda: B.vattn_kept_tiles(g, t()),
        "vattn_sta_fwd": lambda: B.vattn_sta_fwd(g, t(), t(), t(), 0.1, t(), t()),
        "vattn_xwin_fwd": lambda: B.vattn_xwin_fwd(g, 1, t(), t(), t(), 0.1, t(), t()),
        "vattn_xwin_bwd": lambda: B.vattn_xwin_bwd(g, 0, *(t() for _ in range(6)), 0.1, t(), t(), t(), t()),
        "vattn_dual_sym_fwd": lambda: B.vattn_dual_sym_fwd(g, t(), t(), t(), t(), 0.1, t(), workspace=t()),
        "vattn_dual_sym_learned_fwd": lambda: B.vattn_dual_sym_learned_fwd(g, t(), t(), t(), t(), t(), t(), t(), t(), 0.1,
                                                                           t(), t()),
        "vattn_dual_sym_bwd": lambda: B.vattn_dual_sym_bwd(g, *(t() for _ in range(12)), 0.1, t(), t(), t(), t()),
        "vattn_hier_fwd": lambda: B.vattn_hier_fwd(g, t(), t(), t(), 0.1, t(), t(), t()),
        "vattn_hier_bwd": lambda: B.vattn_hier_bwd(g, *(t() for _ in range(6)), 0.1, t(), t(), t(), t()),
        "vattn_sta_fwd_raster": lambda: B.vattn_sta_fwd_raster(g, t(), t(), t(), 0.1, t(), t()),
        "vattn_dual_fwd_fp8": lambda: B.vattn_dual_fwd_fp8(g, t(), t(), t(), t(), 0.1, t(), t()),
        "vattn_sta_fwd_fp8": lambda: B.vattn_sta_fwd_fp8(g, t(), t(), t(), 0.1, t(), t(), t()),
        "vattn_sta_fwd_host": lambda: B.vattn_sta_fwd_host(g, t(**h), t(**h), t(**h), 0.1, t(**h), t(**h), 1, t()),
        "vattn_pool_kv": lambda: B.vattn_pool_kv(g, t(), t(), t(), t()),
        "vattn_global_fwd": lambda: B.vattn_global_fwd(g, t(), t(), t(), 0.1, t(), t()),
        "vattn_dual_fwd": lambda: B.vattn_dual_fwd(g, t(), t(), t(), t(), 0.1, t(), workspace=t()),
        "vattn_dual_fwd_noalloc": lambda: B.vattn_dual_fwd_noalloc(g, t(), t(), t(), t(), 0.1, t()),
        "vattn_sta_bwd": lambda: B.vattn_sta_bwd(g, *(t() for _ in range(6)), 0.1, t(), t(), t(), t()),
        "vattn_dual_bwd": lambda: B.vattn_dual_bwd(g, *(t() for _ in range(11)), 0.1, t(), t(), t(), t(), t()),
        "vattn_get_status": lambda: B.vattn_get_status(),
        "vattn_shutdown": lambda: B.vattn_shutdown(),
        "vattn_debug_set": lambda: B.vattn_debug_set(0, 0),
        "vattn_debug_exp2": lambda: B.vattn_debug_exp2(t(), t()),
        "vattn_debug_query_blocks": lambda: B.vattn_debug_query_blocks(g, 0),
    }


def test_every_wrapper_passes_the_declared_argument_count(B):
    calls = _calls(B)
    for name, call in calls.items():
        B.fake.calls.clear()
        call()
        assert B.fake.calls, name
        for called, args in B.fake.calls:  # one call, or a size query and the call (vattn_debug_query_blocks)
            assert called == name
            assert len(args) == len(B._SIGS[name]), (name, len(args), len(B._SIGS[name]))
    # every C entry point with pointer arguments is exercised above
    declared = {n for n in B._SIGS if n not in ("vattn_workspace_size", "vattn_last_error", "vattn_version")}
    assert declared <= set(calls), declared - set(calls)


def test_workspace_bytes_default_to_the_tensor_size(B):
    g = _geom(B)
    ws = FakeTensor(shape=(12345,), elem=1)
    B.vattn_sta_bwd(g, *(FakeTensor() for _ in range(6)), 0.1, FakeTensor(), FakeTensor(), FakeTensor(), ws)
    (_, args), = B.fake.calls
    assert args[-3] == ws.addr and args[-2] == 12345


def test_placement_and_contiguity_are_checked_before_the_call(B):
    g = _geom(B)
    host = torch.zeros(8)
    with pytest.raises(ValueError, match="host tensor"):
        B.vattn_sta_fwd(g, host, FakeTensor(), FakeTensor(), 0.1, FakeTensor())
    with pytest.raises(ValueError, match="contiguous"):
        B.vattn_sta_fwd(g, FakeTensor(contiguous=False), FakeTensor(), FakeTensor(), 0.1, FakeTensor())
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.vattn_sta_fwd_host(g, FakeTensor(), host, host, 0.1, host, None, 1, FakeTensor())
    with pytest.raises(ValueError, match="contiguous"):
        B.vattn_sta_fwd_host(g, torch.zeros(4, 4).t(), host, host, 0.1, host, None, 1, FakeTensor())
    assert not B.fake.calls
    # raw addresses and None pass through unchanged
    B.vattn_sta_fwd(g, 16, 32, 48, 0.1, 64, None)
    (_, args), = B.fake.calls
    assert args[1:4] == (16, 32, 48) and args[5] == 64 and args[6] is None
    # host tensors are accepted where the C argument is a host pointer
    B.fake.calls.clear()
    B.vattn_sta_fwd_host(g, host, host, host, 0.1, host, None, 1, FakeTensor())
    (_, args), = B.fake.calls
    assert args[1] == host.data_ptr() and args[8] == FakeTensor().addr
