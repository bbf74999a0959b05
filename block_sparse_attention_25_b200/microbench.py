"""Per-call timing of every entry point on one workload, one JSON line per call.

    python -m block_sparse_attention_25_b200.microbench [--config wan14b_720p] [--iters 5]

Each call is timed alone with CUDA events on the launch stream (median of --iters timed
launches after two warm-up launches); inputs are seeded synthetic draws resident in HBM.
Every line carries the call's algorithmic work (bytes for the memory-bound calls, FLOPs for
the contractions), the achieved rate and its fraction of the peak: the measured copy
bandwidth or the measured burst bf16 rate from MEASURED_PEAKS.json at the repository root
(the e4m3 peak is taken as twice the bf16 one, the nominal ratio).
"""
from __future__ import annotations

import argparse
import json
import os

import torch

from . import bsattn as B
from . import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], source="measured")
    return dict(hbm=6650.0, bf16=1590.0, source="fallback")


def _time(fn, iters: int) -> float:
    stream = torch.cuda.current_stream()
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    ms = []
    for _ in range(iters):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    return sorted(ms)[len(ms) // 2]


def schedule_work(row_ptr: torch.Tensor, col_idx: torch.Tensor, s) -> dict:
    """The attention work the forward's schedule performs for given lists, in (64-key kv
    block x query block) pair units: `kept` = the lists' entries; `computed` = what the
    kernel multiplies -- a CTA owns 256 query slots (2 or 4 query blocks in two 128-row
    tiles) and walks the ascending union of its query blocks' lists with both tiles, masking
    for each query block the kv blocks it did not keep, so every query block of the CTA
    pays for every kv block of the union."""
    dev = row_ptr.device
    R, n_kb, n_qb = s.rows, s.n_kb, s.n_qb
    nq = 256 // s.q_block                      # query blocks per CTA
    rp = row_ptr.long()
    nnz = int(rp[-1])
    rows = torch.repeat_interleave(torch.arange(R, device=dev), rp[1:] - rp[:-1])
    keep = torch.zeros(R, n_kb, dtype=torch.bool, device=dev)
    keep[rows, col_idx[:nnz].long()] = True
    bh = s.batch * s.heads
    n_cta = -(-n_qb // nq)
    kp = torch.zeros(bh, n_cta * nq, n_kb, dtype=torch.bool, device=dev)
    kp[:, :n_qb] = keep.view(bh, n_qb, n_kb)
    union = kp.view(bh, n_cta, nq, n_kb).any(2).sum(-1)   # kv blocks each CTA walks
    computed = int(union.sum()) * nq
    return {"kept_pairs": nnz, "computed_pairs": computed,
            "computed_over_kept": round(computed / max(nnz, 1), 4)}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="wan14b_720p")
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--tau", type=float, default=0.99)
    ap.add_argument("--q-clusters", type=int, default=64, help="k-means clusters of the queries")
    ap.add_argument("--k-clusters", type=int, default=256, help="k-means clusters of the keys")
    ap.add_argument("--rounds", type=int, default=10, help="k-means rounds")
    ap.add_argument("--only", choices=["all", "tiles", "semantic", "fwd", "calib", "select"],
                    default="all",
                    help="the 3D-tile path, the semantic-aware permutation path, or both; fwd: "
                         "only the calibration's lists and the forward calls; calib: only "
                         "block_mass and dense_fwd_mass; select: only topp_select on the "
                         "calibration's masses (small profiling cases)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (profiling on a smaller case)")
    args = ap.parse_args(argv)
    build.build()
    dev = torch.device("cuda")
    wl = synth.WORKLOADS[args.config]
    if args.heads is not None:
        wl = wl.scaled(heads=args.heads, name=f"{wl.name}-h{args.heads}")
    s = B.Shape.of(wl)
    pk = _peaks()
    q, k, v = synth.draw_qkv(wl, device=dev)
    e = 2  # bf16 bytes
    S, Np, Hh, D, R, nkb = s.S * s.batch, s.Np * s.batch, s.heads, s.head_dim, s.rows, s.n_kb

    def line(name, ms, work, unit, bound, peak, extra=None):
        rate = work / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
        d = {"call": name, "workload": wl.name, "ms": round(ms, 4), "work": work,
             "work_unit": "bytes" if unit == "GB/s" else "FLOP", "achieved": round(rate, 2),
             "unit": unit, "bound": bound, "peak": peak, "frac": round(rate / peak, 4),
             "peak_source": pk["source"]}
        if extra:
            d.update(extra)
        print(json.dumps(d), flush=True)

    if args.only == "semantic":
        semantic(args, wl, q, k, v, line, pk)
        return
    qt, kt, vt = (B.tile_permute(x, s) for x in (q, k, v))
    if args.only in ("fwd", "calib", "select"):
        return focused(args, wl, s, q, k, v, qt, kt, vt, line, pk)
    out_r = torch.empty_like(q)
    line("tile_permute", _time(lambda: B.tile_permute(q, s, out=qt), args.iters),
         S * Hh * D * e + Np * Hh * D * e, "GB/s", "hbm", pk["hbm"])
    line("tile_permute_inverse", _time(lambda: B.tile_permute(qt, s, inverse=True, out=out_r), args.iters),
         2 * S * Hh * D * e, "GB/s", "hbm", pk["hbm"])
    if D == 128:
        q8 = torch.empty(qt.shape, dtype=torch.uint8, device=dev)
        sc = torch.empty((s.batch, Hh, s.Np // 64), dtype=torch.float32, device=dev)
        line("tile_permute_quant_e4m3",
             _time(lambda: B.tile_permute_quant_e4m3(q, s, out=q8, scales=sc), args.iters),
             S * Hh * D * e + Np * Hh * D + 4 * Hh * Np // 64, "GB/s", "hbm", pk["hbm"])

    mass = torch.empty((s.batch, Hh, s.n_qb, nkb), dtype=torch.float32, device=dev)
    ws_m = B.new_workspace(s, B.OP_BLOCK_MASS, dev)
    qk_pass = 2.0 * Np * s.Np * D * Hh  # one QK^T over all slot pairs
    # The exponential unit binds the calibration: one ex2 per (query slot, key slot) pair of
    # every 256-row tile, against 16 ex2 per clock per SM on 148 SMs at the 1965 MHz maximum.
    n_ex2 = float(s.batch) * Hh * (-(-s.Np // 256) * 256) * s.Np
    ex2_peak = 16.0 * 148 * 1.965e9
    ms_m = _time(lambda: B.block_mass(qt, kt, s, out=mass, ws=ws_m), args.iters)
    line("block_mass", ms_m, qk_pass, "TFLOP/s", "tensor", pk["bf16"],
         {"ex2_per_s": n_ex2 / (ms_m * 1e-3), "ex2_peak_per_s": ex2_peak,
          "ex2_frac": round(n_ex2 / (ms_m * 1e-3) / ex2_peak, 4)})
    out_t = torch.empty_like(qt)
    mass2 = torch.empty_like(mass)
    line("dense_fwd_mass",
         _time(lambda: B.dense_fwd_mass(qt, kt, vt, s, out=out_t, mass=mass2, ws=ws_m), args.iters),
         2 * qk_pass, "TFLOP/s", "tensor", pk["bf16"])  # QK^T and PV once each

    ws_t = B.new_workspace(s, B.OP_TOPP_SELECT, dev)
    row_ptr = torch.empty(R + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(R * nkb, dtype=torch.int32, device=dev)
    ms = _time(lambda: B.topp_select(mass, s, args.tau, ws=ws_t, row_ptr=row_ptr, col_idx=col_idx),
               args.iters)
    nnz = int(row_ptr[-1])
    line("topp_select", ms, 4 * R * nkb + 4 * (R + 1 + nnz), "GB/s", "hbm", pk["hbm"],
         {"kept_fraction": round(nnz / (R * nkb), 5)})

    ws_p = B.new_workspace(s, B.OP_POOLED_MASS, dev)
    pmass = torch.empty_like(mass)
    line("pooled_mass", _time(lambda: B.pooled_mass(qt, kt, s, out=pmass, ws=ws_p), args.iters),
         2 * Np * Hh * D * e + 4 * R * nkb, "GB/s", "hbm", pk["hbm"])

    ws_pt = B.new_workspace(s, B.OP_PATTERN, dev)
    prp = torch.empty(R + 1, dtype=torch.int32, device=dev)
    pci = torch.empty(R * nkb, dtype=torch.int32, device=dev)
    kinds = B.PAT_DIAGONAL | B.PAT_MULTI_DIAGONAL | B.PAT_VERTICAL_STRIPE | B.PAT_SURROUNDING

    def pat():
        B.pattern_csr(s, kinds, diag_width=2, multi_count=2, stripe_stride=16, radius=(1, 2, 2),
                      ws=ws_pt, row_ptr=prp, col_idx=pci, device=dev)
    ms = _time(pat, args.iters)
    pnnz = int(prp[-1])
    line("pattern_csr", ms, 4 * (R + 1 + pnnz), "GB/s", "hbm", pk["hbm"],
         {"kept_fraction": round(pnnz / (R * nkb), 5)})

    ws_f = B.new_workspace(s, B.OP_FWD, dev)
    out_t = torch.empty_like(qt)
    fl = 4.0 * nnz * s.q_block * 64 * D
    work = schedule_work(row_ptr, col_idx, s)
    line("bsattn_fwd", _time(lambda: B.bsattn_fwd(qt, kt, vt, row_ptr, col_idx, s, out=out_t, ws=ws_f),
                             args.iters), fl, "TFLOP/s", "tensor", pk["bf16"],
         {"kept_fraction": round(nnz / (R * nkb), 5), **work})
    # the permutation fused into the forward: raster in, raster out
    out_r = torch.empty_like(q)
    line("bsattn_fwd_raster",
         _time(lambda: B.bsattn_fwd_raster(q, k, v, row_ptr, col_idx, s, out=out_r, ws=ws_f),
               args.iters), fl, "TFLOP/s", "tensor", pk["bf16"],
         {"kept_fraction": round(nnz / (R * nkb), 5)})
    del out_r
    if D == 128:
        k8, v8 = torch.empty_like(q8), torch.empty_like(q8)
        scs = [sc, torch.empty_like(sc), torch.empty_like(sc)]
        B.tile_permute_quant_e4m3(q, s, out=q8, scales=scs[0])
        B.tile_permute_quant_e4m3(k, s, out=k8, scales=scs[1])
        B.tile_permute_quant_e4m3(v, s, out=v8, scales=scs[2])
        line("bsattn_fwd_e4m3",
             _time(lambda: B.bsattn_fwd(q8, k8, v8, row_ptr, col_idx, s, scales=scs, out=out_t, ws=ws_f),
                   args.iters), fl, "TFLOP/s", "tensor", 2 * pk["bf16"],
             {"kept_fraction": round(nnz / (R * nkb), 5)})
    # the same kernel over full lists (every kv block): the dense-path time of the same call
    frp = torch.empty(R + 1, dtype=torch.int32, device=dev)
    fci = torch.empty(R * nkb, dtype=torch.int32, device=dev)
    B.pattern_csr(s, B.PAT_VERTICAL_STRIPE, stripe_stride=1, ws=ws_pt, row_ptr=frp, col_idx=fci,
                  device=dev)
    sparse_ms = _time(lambda: B.bsattn_fwd(qt, kt, vt, row_ptr, col_idx, s, out=out_t, ws=ws_f), args.iters)
    dense_ms = _time(lambda: B.bsattn_fwd(qt, kt, vt, frp, fci, s, out=out_t, ws=ws_f), args.iters)
    line("bsattn_fwd_full_lists", dense_ms, 4.0 * R * nkb * s.q_block * 64 * D, "TFLOP/s", "tensor",
         pk["bf16"], {"kept_fraction": 1.0,
                      "speedup_of_selected_lists": round(dense_ms / sparse_ms, 4)})
    del frp, fci
    # structured lists through the same attention kernel
    pfl = 4.0 * pnnz * s.q_block * 64 * D
    line("bsattn_fwd_pattern", _time(lambda: B.bsattn_fwd(qt, kt, vt, prp, pci, s, out=out_t, ws=ws_f),
                                     args.iters), pfl, "TFLOP/s", "tensor", pk["bf16"],
         {"kept_fraction": round(pnnz / (R * nkb), 5), **schedule_work(prp, pci, s)})
    for w in (ws_m, ws_t, ws_p, ws_pt, ws_f):
        st = B.device_status(w)
        if st != 0:
            raise RuntimeError(f"device status {st}: {B.device_status_words(w)}")
    del qt, kt, vt, out_t, mass, mass2, pmass, col_idx, pci, ws_m, ws_t, ws_p, ws_pt, ws_f
    torch.cuda.empty_cache()
    if args.only == "all":
        semantic(args, wl, q, k, v, line, pk)


def focused(args, wl, s, q, k, v, qt, kt, vt, line, pk):
    """--only fwd: the calibration's lists (untimed), then the tile-major forward (bf16 and,
    for D = 128, e4m3); --only calib: block_mass and dense_fwd_mass; --only select:
    topp_select on the calibration's masses.  Small launch counts for profiler captures."""
    dev = qt.device
    D, Hh, R, nkb = s.head_dim, s.heads, s.rows, s.n_kb
    ws_m = B.new_workspace(s, B.OP_BLOCK_MASS, dev)
    mass = B.block_mass(qt, kt, s, ws=ws_m)
    if args.only == "select":
        ws_t = B.new_workspace(s, B.OP_TOPP_SELECT, dev)
        rp = torch.empty(R + 1, dtype=torch.int32, device=dev)
        ci = torch.empty(R * nkb, dtype=torch.int32, device=dev)
        ms = _time(lambda: B.topp_select(mass, s, args.tau, ws=ws_t, row_ptr=rp, col_idx=ci),
                   args.iters)
        nnz = int(rp[-1])
        line("topp_select", ms, 4 * R * nkb + 4 * (R + 1 + nnz), "GB/s", "hbm", pk["hbm"],
             {"kept_fraction": round(nnz / (R * nkb), 5)})
        ws_m = ws_t
    elif args.only == "calib":
        qk_pass = 2.0 * s.batch * s.Np * s.Np * D * Hh
        line("block_mass", _time(lambda: B.block_mass(qt, kt, s, out=mass, ws=ws_m), args.iters),
             qk_pass, "TFLOP/s", "tensor", pk["bf16"])
        out_t, m2 = torch.empty_like(qt), torch.empty_like(mass)
        line("dense_fwd_mass",
             _time(lambda: B.dense_fwd_mass(qt, kt, vt, s, out=out_t, mass=m2, ws=ws_m), args.iters),
             2 * qk_pass, "TFLOP/s", "tensor", pk["bf16"])
    else:
        rp, ci = B.topp_select(mass, s, args.tau)
        nnz = int(rp[-1])
        fl = 4.0 * nnz * s.q_block * 64 * D
        ws_f = B.new_workspace(s, B.OP_FWD, dev)
        out_t = torch.empty_like(qt)
        line("bsattn_fwd", _time(lambda: B.bsattn_fwd(qt, kt, vt, rp, ci, s, out=out_t, ws=ws_f),
                                 args.iters), fl, "TFLOP/s", "tensor", pk["bf16"],
             {"kept_fraction": round(nnz / (R * nkb), 5), **schedule_work(rp, ci, s)})
        if D == 128:
            q8 = [torch.empty(qt.shape, dtype=torch.uint8, device=dev) for _ in range(3)]
            sc = [torch.empty((s.batch, Hh, s.Np // 64), dtype=torch.float32, device=dev)
                  for _ in range(3)]
            for x, o, c in zip((q, k, v), q8, sc):
                B.tile_permute_quant_e4m3(x, s, out=o, scales=c)
            line("bsattn_fwd_e4m3",
                 _time(lambda: B.bsattn_fwd(q8[0], q8[1], q8[2], rp, ci, s, scales=sc, out=out_t,
                                            ws=ws_f), args.iters),
                 fl, "TFLOP/s", "tensor", 2 * pk["bf16"], {"kept_fraction": round(nnz / (R * nkb), 5)})
        ws_m = ws_f
    st = B.device_status(ws_m)
    if st != 0:
        raise RuntimeError(f"device status {st}: {B.device_status_words(ws_m)}")


def semantic(args, wl, q, k, v, line, pk):
    """The semantic-aware permutation path on the same tokens: k-means of queries and of
    keys, cluster order, cluster-level estimate, top-p over key clusters, attention in
    cluster order, scatter back."""
    s = B.Shape.of(wl)
    Bt, Hh, D, S = s.batch, s.heads, s.head_dim, s.S
    Cq, Ck, rounds = args.q_clusters, args.k_clusters, args.rounds
    cs = B.ClusterShape(Bt, Hh, D, S, Cq, Ck)
    dev = q.device
    g = torch.Generator(device="cpu").manual_seed(17)

    def init_of(x, C):  # C seeded tokens of every head as initial centroids
        pick = torch.randint(0, S, (Bt, Hh, C), generator=g).to(dev)
        xh = x.float().permute(0, 2, 1, 3)                       # [B, Hh, S, D]
        return torch.gather(xh, 2, pick[..., None].expand(-1, -1, -1, D)).contiguous()

    iq, ik = init_of(q, Cq), init_of(k, Ck)
    ws_q = B.new_cluster_workspace(cs, Cq, dev)
    ws_k = B.new_cluster_workspace(cs, Ck, dev)
    cq, ck = iq.clone(), ik.clone()
    lq = torch.empty((Bt, Hh, S), dtype=torch.int32, device=dev)
    nq = torch.empty((Bt, Hh, Cq), dtype=torch.int32, device=dev)
    lk = torch.empty_like(lq)
    nk = torch.empty((Bt, Hh, Ck), dtype=torch.int32, device=dev)
    # fp32 CUDA-core peak: 148 SMs x 128 FMA lanes x 2 FLOP at the boost clock
    alu_peak = 148 * 128 * 2 * 1.965e9 / 1e12

    def km(x, init, cent, C, labels, counts, ws):
        cent.copy_(init)
        B.kmeans(x, cs, C, cent, rounds, labels=labels, counts=counts, ws=ws)
    for name, x, init, cent, C, lab, cnt, ws in (("kmeans_q", q, iq, cq, Cq, lq, nq, ws_q),
                                                 ("kmeans_k", k, ik, ck, Ck, lk, nk, ws_k)):
        ms = _time(lambda: km(x, init, cent, C, lab, cnt, ws), args.iters)
        # distances on the tensor cores as three bf16 products per centroid value: the
        # contraction's peak is a third of the bf16 rate; the round also holds the cluster
        # order and the centroid update
        line(name, ms, 2.0 * Bt * Hh * S * C * D * rounds, "TFLOP/s", "tensor", pk["bf16"] / 3.0,
             {"rounds": rounds, "clusters": C, "ms_per_round": round(ms / rounds, 4),
              "peak_note": "bf16 burst / 3 (hi, mid, lo parts of each centroid)"})
    lay = {}

    def layout():
        lay["q"] = B.cluster_layout(lq, cs, Cq, ws=ws_q)
    ms = _time(layout, args.iters)
    line("cluster_layout", ms, 3 * 4 * Bt * Hh * S, "GB/s", "hbm", pk["hbm"])
    lay["k"] = B.cluster_layout(lk, cs, Ck, ws=ws_k)
    _, sq, tq, _ = lay["q"]
    _, sk, tk, _ = lay["k"]
    qp = torch.empty((Bt, Hh, S, D), dtype=torch.bfloat16, device=dev)
    kp, vp, op = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
    ms = _time(lambda: B.cluster_permute(q, cs, tq, out=qp), args.iters)
    line("cluster_permute", ms, 2 * Bt * Hh * S * D * 2 + 4 * Bt * Hh * S, "GB/s", "hbm", pk["hbm"])
    B.cluster_permute(k, cs, tk, out=kp)
    B.cluster_permute(v, cs, tk, out=vp)
    mass = torch.empty((Bt, Hh, Cq, Ck), dtype=torch.float32, device=dev)
    ms = _time(lambda: B.cluster_mass(cs, cq, nq, ck, nk, out=mass), args.iters)
    line("cluster_mass", ms, 2.0 * Bt * Hh * Cq * Ck * D, "TFLOP/s", "alu", alu_peak)
    rows = Bt * Hh * Cq
    rp = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    ci = torch.empty(rows * Ck, dtype=torch.int32, device=dev)
    ms = _time(lambda: B.topp_select_rows(mass, args.tau, row_ptr=rp, col_idx=ci), args.iters)
    nnz = int(rp[-1])
    line("topp_select_rows", ms, 4 * rows * Ck + 4 * (rows + 1 + nnz), "GB/s", "hbm", pk["hbm"],
         {"kept_fraction": round(nnz / (rows * Ck), 5)})
    # algorithmic FLOPs: every (query, key) pair of the selected cluster pairs, 4 D each
    rpc, cic = rp.cpu().long(), ci[:nnz].cpu().long()
    nqc, nkc = nq.cpu().long().view(-1), nk.cpu().long().view(Bt * Hh, Ck)
    head = torch.arange(rows) // Cq
    sel_keys = torch.zeros(rows, dtype=torch.long)
    for r in range(rows):
        sel_keys[r] = nkc[head[r], cic[rpc[r]:rpc[r + 1]]].sum()
    pairs = float((nqc * sel_keys).sum())
    ws_f = B.new_cluster_fwd_workspace(cs, dev)
    ms = _time(lambda: B.cluster_fwd(qp, kp, vp, cs, sq, nq, sk, nk, rp, ci, out=op, ws=ws_f),
               args.iters)
    line("cluster_fwd", ms, 4.0 * D * pairs, "TFLOP/s", "tensor", pk["bf16"],
         {"kept_pair_fraction": round(pairs / (Bt * Hh * float(S) * S), 5)})
    out = torch.empty_like(q)
    ms = _time(lambda: B.cluster_permute(op, cs, tq, inverse=True, out=out), args.iters)
    line("cluster_permute_inverse", ms, 2 * Bt * Hh * S * D * 2 + 4 * Bt * Hh * S, "GB/s", "hbm",
         pk["hbm"])
    for w in (ws_q, ws_k, ws_f):
        st = B.device_status(w)
        if st != 0:
            raise RuntimeError(f"device status {st}: {B.device_status_words(w)}")


if __name__ == "__main__":
    main()
