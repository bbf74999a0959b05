"""Shape validation of the C ABI against the limits include/bsattn.h documents, on 4,000
seeded random shapes (valid and invalid, near every limit).  No GPU: the library sizes
workspaces and rejects shapes on the host.

The documented rules: batch, heads, head_dim, T, H, W >= 1; Tp, Hp, Wp multiples of 4
covering T, H, W; Np = Tp*Hp*Wp < 2^30 and a multiple of q_block; head_dim in {64, 128};
q_block in {64, 128}; kv_block = 64; R = B*Hh*(Np/q_block) < 2^31; Np/64 <= 4096;
R*(Np/64) < 2^31.  Inconsistent extents are INVALID_ARG, consistent shapes beyond the
limits UNSUPPORTED, and bsa_workspace_bytes is 0 for both.
"""
import ctypes

import numpy as np
import pytest
import torch

FAKE = ctypes.c_void_p(0x10000)   # aligned, never dereferenced: every call fails on the host


@pytest.fixture(scope="module")
def B():
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    b.lib()
    return b


def _violations(d):
    """(inconsistent, beyond_limits) flags of a shape, from the documented rules."""
    inconsistent = (min(d["batch"], d["heads"], d["head_dim"], d["T"], d["H"], d["W"]) < 1
                    or d["Tp"] < d["T"] or d["Hp"] < d["H"] or d["Wp"] < d["W"]
                    or d["Tp"] % 4 or d["Hp"] % 4 or d["Wp"] % 4)
    np_ = d["Tp"] * d["Hp"] * d["Wp"]
    limits = (np_ >= 2 ** 30 or d["head_dim"] not in (64, 128) or d["kv_block"] != 64
              or d["q_block"] not in (64, 128))
    if not inconsistent and not limits:
        if np_ % d["q_block"]:
            inconsistent = True
        else:
            rows = d["batch"] * d["heads"] * (np_ // d["q_block"])
            limits = rows >= 2 ** 31 or np_ // 64 > 4096 or rows * (np_ // 64) >= 2 ** 31
    return bool(inconsistent), bool(limits)


def _random_shape(rng):
    """A valid shape (grids up to the 4096-kv-block limit and beyond), then with probability
    3/4 one field moved to a value near or past a documented limit."""
    T, H, W = (int(rng.integers(1, 70)) for _ in range(3))
    d = dict(batch=int(rng.integers(1, 4)), heads=int(rng.choice([1, 2, 12, 40])),
             head_dim=int(rng.choice([64, 128])), T=T, H=H, W=W,
             Tp=-(-T // 4) * 4, Hp=-(-H // 4) * 4, Wp=-(-W // 4) * 4,
             q_block=int(rng.choice([64, 128])), kv_block=64)
    if d["q_block"] == 128 and (d["Tp"] * d["Hp"] * d["Wp"]) % 128:
        d["Wp"] += 4 if (d["Wp"] // 4) % 2 else 0          # make Np a multiple of 128
        if (d["Tp"] * d["Hp"] * d["Wp"]) % 128:
            d["q_block"] = 64
    if rng.random() < 0.75:
        f = str(rng.choice(["batch", "heads", "head_dim", "T", "Tp", "Wp", "q_block",
                            "kv_block", "big", "huge"]))
        if f == "batch":
            d["batch"] = int(rng.choice([-1, 0, 1 << 20, 1 << 30]))
        elif f == "heads":
            d["heads"] = int(rng.choice([0, -3, 1 << 16, 1 << 24]))
        elif f == "head_dim":
            d["head_dim"] = int(rng.choice([0, 32, 96, 256]))
        elif f == "T":
            d["T"] = int(rng.choice([0, -1, d["Tp"] + 1]))
        elif f == "Tp":
            d["Tp"] += int(rng.choice([1, 2, -4]))
        elif f == "Wp":
            d["Wp"] += int(rng.choice([4, 8, 3]))
        elif f == "q_block":
            d["q_block"] = int(rng.choice([32, 100, 256]))
        elif f == "kv_block":
            d["kv_block"] = int(rng.choice([32, 128]))
        elif f == "big":                                   # near the 4096-kv-block limit
            d.update(T=61, H=62, W=int(rng.choice([61, 64, 65, 68])), Tp=64, Hp=64)
            d["Wp"] = -(-d["W"] // 4) * 4
        else:                                              # near Np = 2^30
            d.update(T=1024, H=1024, W=1020, Tp=1024, Hp=1024, Wp=int(rng.choice([1020, 1024])))
    return d


def test_workspace_sizes_follow_the_documented_limits(B):
    rng = np.random.default_rng(77)
    n_valid = n_bad = 0
    for _ in range(4000):
        d = _random_shape(rng)
        inconsistent, limits = _violations(d)
        size = B.workspace_bytes(B.Shape(**d), B.OP_FWD)
        if inconsistent or limits:
            assert size == 0, d
            n_bad += 1
        else:
            assert size >= 256, d
            n_valid += 1
    assert n_valid > 200 and n_bad > 1000


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake-pointer validation checks run on hosts without a GPU only")
def test_status_codes_follow_the_documented_classes(B):
    """bsa_pooled_mass with aligned fake pointers and no workspace: a valid shape gets as far
    as the workspace check (CAPACITY); an invalid one returns its class first."""
    L = B.lib()
    rng = np.random.default_rng(78)
    seen = set()
    for _ in range(4000):
        d = _random_shape(rng)
        inconsistent, limits = _violations(d)
        st = L.bsa_pooled_mass(ctypes.byref(B.Shape(**d).c()), FAKE, FAKE, ctypes.c_float(0.088),
                               FAKE, FAKE, 0, None)
        if not inconsistent and not limits:
            assert st == 3, (d, st)
        elif inconsistent and not limits:
            assert st == 1, (d, st)
        elif limits and not inconsistent:
            assert st == 2, (d, st)
        else:
            assert st in (1, 2), (d, st)
        seen.add(st)
    assert seen == {1, 2, 3}


def _cluster_valid(d):
    if min(d["batch"], d["heads"], d["n_tokens"], d["n_q_clusters"], d["n_k_clusters"]) < 1:
        return False
    if d["head_dim"] not in (64, 128) or d["n_tokens"] > 2 ** 24:
        return False
    if d["n_q_clusters"] > 1024 or d["n_k_clusters"] > 1024:
        return False
    bh = d["batch"] * d["heads"]
    return (bh * d["n_tokens"] * (d["head_dim"] // 8) < 2 ** 31
            and bh * d["n_q_clusters"] * d["n_k_clusters"] < 2 ** 31)


def test_cluster_workspace_sizes_follow_the_documented_limits(B):
    rng = np.random.default_rng(79)
    n_valid = n_bad = 0
    for _ in range(3000):
        d = dict(batch=int(rng.choice([0, 1, 1, 2, 4, 1 << 12])),
                 heads=int(rng.choice([-1, 1, 2, 40, 1 << 10])),
                 head_dim=int(rng.choice([32, 64, 64, 128, 128, 256])),
                 n_tokens=int(rng.choice([0, 1, 300, 75600, 1 << 20, 1 << 24, (1 << 24) + 1])),
                 n_q_clusters=int(rng.choice([0, 1, 64, 1024, 1025])),
                 n_k_clusters=int(rng.choice([1, 256, 1024, 2048])))
        cs = B.ClusterShape(**d)
        got = B.lib().bsa_cluster_fwd_workspace_bytes(ctypes.byref(cs.c()))
        km = B.lib().bsa_kmeans_workspace_bytes(ctypes.byref(cs.c()), int(d["n_q_clusters"]))
        if _cluster_valid(d):
            assert got >= 256 and km >= 256, d
            n_valid += 1
        else:
            assert got == 0 and km == 0, d
            n_bad += 1
    assert n_valid > 100 and n_bad > 500
