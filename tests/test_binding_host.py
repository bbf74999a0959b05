"""The Python binding's argument checks, on the CPU.

Every tensor the binding hands to the library as a raw pointer must be a contiguous CUDA
tensor of the right dtype and size: a host tensor there would reach a kernel as a device
address.  Two halves:
- with the real device check, host tensors (inputs, outputs, workspaces, lists) are refused
  with TypeError / ValueError before anything is called;
- with the device check and the library stubbed, the call patterns the bench, the
  microbench and the GPU tests use (outputs, workspaces and lists they allocate themselves)
  are all accepted, so the checks reject no legitimate call.
"""
import pytest
import torch

from block_sparse_attention_25_b200 import bsattn as bs
from block_sparse_attention_25_b200 import synth


class _StubLib:
    """Every bsa_* call returns 0 (BSA_OK); workspace-size queries return 4096 bytes."""

    calls = []

    def __getattr__(self, name):
        def call(*args):
            _StubLib.calls.append(name)
            return 4096 if name.endswith("workspace_bytes") else 0
        return call


@pytest.fixture
def stub(monkeypatch):
    _StubLib.calls = []
    monkeypatch.setattr(bs, "lib", lambda: _StubLib())
    monkeypatch.setattr(bs, "_stream", lambda stream=None: None)
    return _StubLib


@pytest.fixture
def as_device(stub, monkeypatch):
    monkeypatch.setattr(bs, "_is_device", lambda t: True)
    return stub


def _shape():
    return bs.Shape.of(synth.WORKLOADS["tiny"].scaled(storage="bf16"))


def _tensors(s):
    raster = (s.batch, s.S, s.heads, s.head_dim)
    tiled = (s.batch, s.heads, s.Np, s.head_dim)
    return dict(
        q=torch.zeros(raster, dtype=torch.bfloat16),
        qt=torch.zeros(tiled, dtype=torch.bfloat16),
        q8=torch.zeros(tiled, dtype=torch.uint8),
        sc=torch.ones((s.batch, s.heads, s.Np // 64), dtype=torch.float32),
        mass=torch.zeros((s.batch, s.heads, s.n_qb, s.n_kb), dtype=torch.float32),
        rp=torch.zeros(s.rows + 1, dtype=torch.int32),
        ci=torch.zeros(s.rows * s.n_kb, dtype=torch.int32),
        out_t=torch.zeros(tiled, dtype=torch.bfloat16),
        out_r=torch.zeros(raster, dtype=torch.bfloat16),
        ws=torch.zeros(4096, dtype=torch.uint8),
    )


def test_the_stubbed_patterns_are_accepted(as_device):
    """The argument patterns of the bench, the microbench and the GPU tests."""
    s = _shape()
    t = _tensors(s)
    bs.tile_permute(t["q"], s, out=t["qt"])
    bs.tile_permute(t["out_t"], s, inverse=True, out=t["out_r"])
    bs.tile_permute_quant_e4m3(t["q"], s, out=t["q8"], scales=t["sc"])
    bs.tile_permute_quant_e4m3(t["q"], s)
    bs.block_mass(t["qt"], t["qt"], s, out=t["mass"], ws=t["ws"])
    bs.block_mass(t["qt"], t["qt"], s)
    bs.dense_fwd_mass(t["qt"], t["qt"], t["qt"], s, out=t["out_t"], mass=t["mass"], ws=t["ws"])
    bs.dense_fwd_mass(t["qt"], t["qt"], t["qt"], s, want_lse=True)
    bs.pooled_mass(t["qt"], t["qt"], s, out=t["mass"], ws=t["ws"])
    bs.topp_select(t["mass"], s, 0.99, ws=t["ws"], row_ptr=t["rp"], col_idx=t["ci"])
    bs.topp_select(t["mass"], s, 1.0, col_capacity=3, ws=t["ws"])
    bs.topp_select_noalloc(t["mass"], s, 0.99, status=torch.zeros(4, dtype=torch.int32))
    bs.pattern_csr(s, bs.PAT_VERTICAL_STRIPE, stripe_stride=1, ws=t["ws"], row_ptr=t["rp"],
                   col_idx=t["ci"], device="cpu")
    bs.bsattn_fwd(t["qt"], t["qt"], t["qt"], t["rp"], t["ci"], s, out=t["out_t"], ws=t["ws"])
    bs.bsattn_fwd(t["qt"], t["qt"], t["qt"], t["rp"], t["ci"][:1], s, want_lse=True)
    bs.bsattn_fwd(t["q8"], t["q8"], t["q8"], t["rp"], t["ci"], s, scales=(t["sc"],) * 3,
                  out=t["out_t"], ws=t["ws"])
    bs.bsattn_fwd_raster(t["q"], t["q"], t["q"], t["rp"], t["ci"], s, out=t["out_r"], ws=t["ws"])
    lse = torch.full((s.batch, s.heads, s.S), float("nan"))
    bs.bsattn_fwd_raster(t["q"], t["q"], t["q"], t["rp"], t["ci"], s, want_lse=True,
                         out=t["out_r"], lse=lse, ws=t["ws"][:2048])
    bs.topp_select_rows(torch.zeros((6, 9), dtype=torch.float32), 0.95)
    cs = bs.ClusterShape(1, 2, 64, 300, 4, 5)
    x = torch.zeros((1, 300, 2, 64), dtype=torch.bfloat16)
    xc = torch.zeros((1, 2, 300, 64), dtype=torch.bfloat16)
    init = torch.zeros((1, 2, 4, 64), dtype=torch.float32)
    bs.kmeans(x, cs, 4, init, 2)
    bs.kmeans(x, cs, 4, init, 2, labels=torch.zeros((1, 2, 300), dtype=torch.int32),
              counts=torch.zeros((1, 2, 4), dtype=torch.int32), ws=t["ws"])
    labels = torch.zeros((1, 2, 300), dtype=torch.int32)
    bs.cluster_layout(labels, cs, 4)
    bs.cluster_permute(x, cs, labels)
    bs.cluster_permute(xc, cs, labels, inverse=True, out=torch.zeros_like(x))
    qc, kc = torch.zeros((1, 2, 4, 64)), torch.zeros((1, 2, 5, 64))
    qn, kn = torch.zeros((1, 2, 4), dtype=torch.int32), torch.zeros((1, 2, 5), dtype=torch.int32)
    bs.cluster_mass(cs, qc, qn, kc, kn)
    bs.cluster_mass(cs, qc, qn, kc, kn, out=torch.zeros((1, 2, 4, 5)))
    bs.topp_select_rows(torch.zeros((8, 5)), 0.9, row_ptr=torch.zeros(9, dtype=torch.int32),
                        col_idx=torch.zeros(40, dtype=torch.int32))
    bs.cluster_layout(labels, cs, 4, ws=t["ws"])
    bs.cluster_permute(x, cs, labels, out=torch.zeros_like(xc))
    crp = torch.zeros(1 * 2 * 4 + 1, dtype=torch.int32)
    bs.cluster_fwd(xc, xc, xc, cs, qn, qn, kn, kn, crp, torch.zeros(1, dtype=torch.int32),
                   out=torch.full_like(xc, 7.0), ws=torch.zeros(4096, dtype=torch.uint8))
    names = set(as_device.calls)
    for n in ("bsa_tile_permute", "bsa_tile_permute_quant_e4m3", "bsa_block_mass",
              "bsa_dense_fwd_mass", "bsa_pooled_mass", "bsa_topp_select",
              "bsa_topp_select_noalloc", "bsa_pattern_csr", "bsa_fwd", "bsa_fwd_raster",
              "bsa_topp_select_rows", "bsa_kmeans", "bsa_cluster_layout", "bsa_cluster_permute",
              "bsa_cluster_mass", "bsa_cluster_fwd"):
        assert n in names, n


def _refused_host(fn, *a, allow_clear=False, **kw):
    """fn raises TypeError / ValueError having called nothing but size queries (and, when
    allow_clear, the status clear of a workspace it allocated on the device itself)."""
    before = len(_StubLib.calls)
    with pytest.raises((TypeError, ValueError)):
        fn(*a, **kw)
    allowed = ("bsa_clear_status",) if allow_clear else ()
    compute = [c for c in _StubLib.calls[before:]
               if not c.endswith("workspace_bytes") and c not in allowed]
    assert compute == [], compute


def test_host_buffers_are_refused_before_any_call(stub):
    """The real device check: every CPU tensor the library would dereference is refused."""
    _refused = _refused_host
    s = _shape()
    t = _tensors(s)
    _refused(bs.tile_permute, t["q"], s)
    _refused(bs.block_mass, t["qt"], t["qt"], s)
    _refused(bs.bsattn_fwd, t["qt"], t["qt"], t["qt"], t["rp"], t["ci"], s)
    _refused(bs.topp_select, t["mass"], s, 0.99)
    _refused(bs.topp_select_rows, torch.zeros((6, 9)), 0.9)
    _refused(bs.pattern_csr, s, bs.PAT_DIAGONAL, device="cpu")
    _refused(bs.selftest_wait, torch.zeros(256, dtype=torch.uint8))
    _refused(bs.new_workspace, s, bs.OP_FWD, "cpu")
    _refused(bs.clear_status, torch.zeros(256, dtype=torch.uint8))


def test_bad_outputs_and_workspaces_are_refused(as_device, monkeypatch):
    """Outputs, lists and workspaces the caller passes: wrong dtype, wrong shape, too few
    elements, not contiguous, or on the host (device check restored for the last)."""
    s = _shape()
    t = _tensors(s)
    qt = t["qt"]

    def _refused(fn, *a, **kw):
        _refused_host(fn, *a, allow_clear=True, **kw)

    _refused(bs.block_mass, qt, qt, s, out=t["mass"].double())
    _refused(bs.block_mass, qt, qt, s, out=t["mass"][..., :-1])
    _refused(bs.block_mass, qt, qt, s, ws=torch.zeros(1024, dtype=torch.float32))
    _refused(bs.dense_fwd_mass, qt, qt, qt, s, out=t["out_t"].float())
    _refused(bs.pooled_mass, qt, qt, s, out=t["mass"].transpose(-1, -2))
    _refused(bs.topp_select, t["mass"], s, 0.99, col_idx=t["ci"][:5])
    _refused(bs.topp_select, t["mass"], s, 0.99, row_ptr=t["rp"][:-1])
    _refused(bs.topp_select_noalloc, t["mass"], s, 0.99, status=torch.zeros(2, dtype=torch.int32))
    _refused(bs.topp_select_noalloc, t["mass"], s, 0.99, status=torch.zeros(4, dtype=torch.float32))
    _refused(bs.pattern_csr, s, bs.PAT_DIAGONAL, col_idx=t["ci"][:3], device="cpu")
    _refused(bs.bsattn_fwd, qt, qt, qt, t["rp"], t["ci"], s, out=t["out_r"])
    _refused(bs.bsattn_fwd, qt, qt, qt, t["rp"], t["ci"].long(), s)
    _refused(bs.bsattn_fwd, qt, qt, qt, t["rp"], t["ci"], s, want_lse=True,
             lse=torch.zeros(3, dtype=torch.float32))
    _refused(bs.bsattn_fwd_raster, t["q"], t["q"], t["q"], t["rp"], t["ci"], s, out=t["out_t"])
    _refused(bs.tile_permute_quant_e4m3, t["q"], s, scales=t["sc"][..., :-1])
    wide = torch.zeros((s.batch, s.heads, s.Np, 2 * s.head_dim), dtype=torch.bfloat16)
    _refused(bs.bsattn_fwd, qt, qt, qt, t["rp"], t["ci"], s, out=wide[..., :s.head_dim])
    monkeypatch.setattr(bs, "_is_device", lambda x: x is not t["ws"])
    _refused(bs.bsattn_fwd, qt, qt, qt, t["rp"], t["ci"], s, ws=t["ws"])
