"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances (stated by the workload definitions): bf16 layers match the fp64
oracle within 2e-2 max-abs, fp32 layers within 1e-4.  Selected block sets must
be identical except where the oracle's k-th selected importance and the
importance of a swapped block differ by less than 1e-3 relative; rows with such
a swap are compared against the oracle run on the kernel's own selection.
"""
from __future__ import annotations

import numpy as np

import oracle
from sparse_attention_long_block_b200.inputs import Workload, generate

TOL = {"bf16": 2e-2, "fp32": 1e-4}
TIE_REL = 1e-3


def oracle_params(wl: Workload) -> oracle.OracleParams:
    return oracle.OracleParams(h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                               top_k=wl.top_k, window=wl.window,
                               round_cmp_bf16=(wl.dtype == "bf16"), stride=wl.stride or None)


def stratified_rows(is_vision: np.ndarray, block: int = 64, every: int = 97,
                    first: int = 128, max_text: int | None = None, seed: int = 0):
    """Global positions to check at large sizes: the first vision rows, every
    `every`-th vision row, rows on both sides of block boundaries, and the text
    rows (all, or an evenly spread subset of max_text)."""
    vis = np.nonzero(is_vision)[0]
    txt = np.nonzero(is_vision == 0)[0]
    nv = len(vis)
    ranks = set(range(min(first, nv)))
    ranks.update(range(0, nv, every))
    rng = np.random.default_rng(seed)
    nblk = nv // block
    for j in rng.choice(np.arange(1, max(2, nblk)), size=min(24, max(1, nblk - 1)), replace=False):
        for x in (j * block - 1, j * block):
            if 0 <= x < nv:
                ranks.add(int(x))
    if nv:
        ranks.add(nv - 1)
    rows = [int(vis[r]) for r in sorted(ranks)]
    if max_text is not None and len(txt) > max_text:
        txt = txt[np.linspace(0, len(txt) - 1, max_text).astype(int)]
    rows += [int(t) for t in txt]
    return np.array(sorted(rows), dtype=np.int32)


def run_gpu(wl: Workload, x: dict, want=(), forced_idx=None, ranks=None, cmp_mlp=None):
    """Run the CUDA layer through the C ABI; returns numpy results.  With
    `ranks`, the per-vision-rank exports (idx, imp) are cut to those ranks on
    the device before the copy to the host; with `cmp_mlp` (weights dict) the
    compression branch uses that perceptron."""
    import torch
    from sparse_attention_long_block_b200 import binding
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dev = "cuda"
    q = torch.from_numpy(x["q"]).to(dev, td).contiguous()
    k = torch.from_numpy(x["k"]).to(dev, td).contiguous()
    v = torch.from_numpy(x["v"]).to(dev, td).contiguous()
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype, stride=wl.stride)
    if cmp_mlp is not None:
        layer.set_cmp_mlp({nm: torch.from_numpy(a) for nm, a in cmp_mlp.items()})
    fidx = None
    if forced_idx is not None:
        fidx = torch.from_numpy(np.ascontiguousarray(forced_idx, np.int32)).to(dev)
    dbg, tens = binding.make_debug(wl.n, wl.h_q, wl.h_kv, wl.d, wl.top_k, wl.block, dtype=td,
                                   want=want, forced_idx=fidx, stride=wl.stride)
    out = layer.forward(q, k, v, isv, gate, dbg=dbg if (want or fidx is not None) else None)
    torch.cuda.synchronize()
    status = layer.device_status()
    res = {"out": out.float().cpu().numpy(), "status": status,
           "counts": layer.counts(), "launches": layer.launches()}
    for name, t in tens.items():
        if name == "forced_idx":
            continue
        if ranks is not None and name in ("idx", "imp"):
            t = t[:, torch.as_tensor(ranks, device=t.device, dtype=torch.long), :]
        res[name] = t.float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()
    layer.close()
    return res


def expected_candidates(i, block, force_first=True, force_local=True):
    """The blocks a vision query of rank i may select, and the forced ones
    ("VideoNSA: Native Sparse Attention Scales Video Understanding", paper
    notes, section "Method", read as: the complete blocks at or before i,
    plus block 0 and the query's own block, which are always kept)."""
    forced = set()
    if force_first:
        forced.add(0)
    if force_local:
        forced.add(i // block)
    visible = set(range((i + 1) // block))
    return visible | forced, forced


def check_selection_row(row, i, top_k, block, force_first=True, force_local=True,
                        expect_count=None):
    """Structure of one exported selection row [top_k] of the vision query of
    rank i: the selected blocks strictly ascending (so duplicate-free), then -1
    padding only; exactly min(top_k, #candidates) entries (or `expect_count`);
    every entry a candidate; every forced block present.  Raises on a
    violation; returns the selected blocks as a list."""
    row = [int(j) for j in row]
    cands, forced = expected_candidates(i, block, force_first, force_local)
    n_valid = 0
    while n_valid < len(row) and row[n_valid] >= 0:
        n_valid += 1
    sel = row[:n_valid]
    if any(j != -1 for j in row[n_valid:]):
        raise AssertionError(f"rank {i}: entries after the first -1 are not all -1: {row}")
    if any(b <= a for a, b in zip(sel, sel[1:])):
        raise AssertionError(f"rank {i}: selection not strictly ascending: {row}")
    want = min(top_k, len(cands)) if expect_count is None else expect_count
    if n_valid != want:
        raise AssertionError(f"rank {i}: {n_valid} blocks selected, expected {want}: {row}")
    bad = [j for j in sel if j not in cands]
    if bad:
        raise AssertionError(f"rank {i}: blocks {bad} are not visible to the query: {row}")
    missing = sorted(forced - set(sel))
    if missing:
        raise AssertionError(f"rank {i}: forced blocks {missing} missing: {row}")
    return sel


def check_selection(gpu_idx_rows, ora_idx, ora_imp, top_k, force_first=True,
                    force_local=True, block=64, ranks=None):
    """gpu_idx_rows, ora_idx: [R][G][k]; ora_imp [R][G][nb]; ranks [R] the
    vision ranks of the rows (required).  Every GPU row must be a well-formed
    selection (check_selection_row) with as many blocks as the oracle's row.
    Returns the row indices (into R) whose block set differs from the
    oracle's within the tie band; raises on a difference outside it."""
    if ranks is None:
        raise ValueError("check_selection needs the vision ranks of the rows")
    swapped = []
    R, G, _ = ora_idx.shape
    for r in range(R):
        i = int(ranks[r])
        _, forced = expected_candidates(i, block, force_first, force_local)
        for g in range(G):
            b_list = check_selection_row(ora_idx[r, g], i, top_k, block, force_first,
                                         force_local)
            a_list = check_selection_row(gpu_idx_rows[r, g], i, top_k, block, force_first,
                                         force_local, expect_count=len(b_list))
            a, b = set(a_list), set(b_list)
            if a == b:
                continue
            chosen = [j for j in b if j not in forced]
            if not chosen:
                raise AssertionError(f"row {r} group {g}: sets differ {sorted(a ^ b)} "
                                     "with no free slot in the oracle's choice")
            s_k = min(ora_imp[r, g, j] for j in chosen)
            for j in a ^ b:
                if j in forced or j >= ora_imp.shape[2]:
                    raise AssertionError(f"row {r} group {g}: forced/invalid block {j} differs")
                if abs(ora_imp[r, g, j] - s_k) > TIE_REL * abs(s_k):
                    raise AssertionError(
                        f"row {r} group {g}: block {j} imp {ora_imp[r, g, j]:.8g} vs k-th "
                        f"{s_k:.8g} outside the tie band; gpu {sorted(a)} oracle {sorted(b)}")
            swapped.append(r)
    return sorted(set(swapped))


def compare_layer(wl: Workload, x: dict, rows=None, want_branches=True, check_imp=True,
                  cmp_mlp=None):
    """Full comparison of the CUDA layer with the oracle on `rows` (all if
    None), optionally with a compression perceptron.  Returns a dict of error
    statistics."""
    p = oracle_params(wl)
    want = ("idx", "imp") + (("o_cmp", "o_slc", "o_swa") if want_branches else ())
    isv = x["is_vision"]
    if rows is None:
        rows = np.arange(wl.n, dtype=np.int32)
    rank_of = -np.ones(wl.n, np.int64)
    vis = np.nonzero(isv)[0]
    rank_of[vis] = np.arange(len(vis))
    ranks = rank_of[rows]
    is_v = ranks >= 0
    vr = ranks[is_v]
    g = run_gpu(wl, x, want=want + (("lse_cmp",) if want_branches else ()), ranks=vr,
                cmp_mlp=cmp_mlp)
    assert g["status"] == 0, f"device status {g['status']}"
    nv_gpu, nt_gpu = g["counts"]
    assert nv_gpu == int(isv.sum()) and nt_gpu == len(isv) - int(isv.sum())
    o = oracle.forward(p, x["q"], x["k"], x["v"], isv, x["gate"], x["w_k"], x["w_v"],
                       rows=rows, want=want + ("lse_cmp",), cmp_mlp=cmp_mlp)
    tol = TOL[wl.dtype]
    stats = {}
    # selection sets (g["idx"], g["imp"] are already cut to the ranks vr)
    if is_v.any():
        gidx = np.transpose(g["idx"], (1, 0, 2))
        swapped_local = check_selection(gidx, o["idx"][is_v], o["imp"][is_v], wl.top_k,
                                        block=wl.block, ranks=vr)
        stats["swapped_rows"] = len(swapped_local)
        if check_imp and o["nb"] > 0:
            gimp = np.transpose(g["imp"][:, :, :o["nb"]], (1, 0, 2))
            nvis = np.minimum((vr + 1) // wl.block, o["nb"])
            mask = np.arange(o["nb"])[None, :] < nvis[:, None]
            err = np.abs(gimp - o["imp"][is_v]) * mask[:, None, :]
            stats["imp_max_abs"] = float(err.max())
            assert stats["imp_max_abs"] < (1e-3 if wl.dtype == "bf16" else 1e-5), stats
    else:
        swapped_local = []
    ref_out = o["out"].copy()
    if swapped_local:
        sub = np.nonzero(is_v)[0][swapped_local]
        fidx = np.transpose(g["idx"][:, swapped_local, :], (1, 0, 2))
        o2 = oracle.forward(p, x["q"], x["k"], x["v"], isv, x["gate"], x["w_k"], x["w_v"],
                            rows=rows[sub], forced_idx=fidx, want=("o_slc",), cmp_mlp=cmp_mlp)
        ref_out[sub] = o2["out"]
        if "o_slc" in o:
            o["o_slc"][sub] = o2["o_slc"]
    gout = g["out"][rows]
    err = np.abs(gout - ref_out)
    stats["out_max_abs"] = float(err.max()) if err.size else 0.0
    stats["rows"] = int(len(rows))
    assert np.isfinite(gout).all()
    assert stats["out_max_abs"] <= tol, stats
    if want_branches and is_v.any():
        vrows = rows[is_v]
        for name in ("o_cmp", "o_slc", "o_swa"):
            e = np.abs(g[name][vrows] - o[name][is_v])
            stats[name + "_max_abs"] = float(e.max())
            assert stats[name + "_max_abs"] <= tol, (name, stats)
        lse_g = g["lse_cmp"][ranks[is_v]]
        lse_o = o["lse_cmp"][is_v]
        fin = np.isfinite(lse_o)
        assert np.array_equal(np.isfinite(lse_g), fin)
        if fin.any():
            stats["lse_max_abs"] = float(np.abs(lse_g[fin] - lse_o[fin]).max())
            assert stats["lse_max_abs"] < (2e-3 if wl.dtype == "bf16" else 1e-5), stats
    return stats


def compare_pool(wl: Workload, x: dict, cmp_mlp=None):
    p = oracle_params(wl)
    kc, vc = oracle.pool_proj(p, x["k"], x["v"], x["is_vision"], x["w_k"], x["w_v"],
                              cmp_mlp=cmp_mlp)
    g = run_gpu(wl, x, want=("k_cmp", "v_cmp"), cmp_mlp=cmp_mlp)
    nb = kc.shape[0]  # compression blocks (they overlap when the stride is below the block)
    out = {}
    stride = wl.stride or wl.block
    allv = np.nonzero(x["is_vision"])[0]
    vis = np.concatenate([allv[c * stride: c * stride + wl.block] for c in range(nb)]) \
        if nb else allv[:0]
    for name, ref, src, w in (("k_cmp", kc, x["k"], x["w_k"]), ("v_cmp", vc, x["v"], x["w_v"])):
        got = g[name][:nb].astype(np.float64)
        if wl.dtype == "bf16":
            # both sides round once to bf16: they may differ by one bf16 ulp where
            # the fp32 accumulation and the exact value straddle a rounding midpoint.
            # Where the block mean and the projection cancel, the fp32 error of
            # the B-term sum and the d-term product, (B + d) 2^-24 (mean|x|).|W|,
            # can exceed that ulp of the (small) exact value; the bf16 rounding of
            # the fp32 result then adds one more ulp.
            mabs = np.abs(src[vis].astype(np.float64)).reshape(nb, wl.block, wl.h_kv, wl.d).mean(1)
            if cmp_mlp is None:
                acc = (wl.block + wl.d) * 2.0 ** -24 * (mabs @ np.abs(w.astype(np.float64)))
            else:
                # perceptron: |SiLU(z)| <= |z| and |SiLU'| <= 1.1 bound the hidden
                # layer by A1 = mean|x|.|W1| + |b1| and its fp32 error (sum, product,
                # exp) by (1.1 (B + d) 2^-24 + 2^-22) A1; the second product adds
                # (H + 1) 2^-24 (A1.|W2| + |b2|)
                t = name[0]
                w1 = np.abs(cmp_mlp["w1_" + t].astype(np.float64))
                w2 = np.abs(cmp_mlp["w2_" + t].astype(np.float64))
                b1 = np.abs(cmp_mlp["b1_" + t].astype(np.float64))
                b2 = np.abs(cmp_mlp["b2_" + t].astype(np.float64))
                hid = w1.shape[1]
                a1 = mabs @ w1 + b1
                e_h = (1.1 * (wl.block + wl.d) * 2.0 ** -24 + 2.0 ** -22) * a1
                acc = e_h @ w2 + (hid + 1) * 2.0 ** -24 * (a1 @ w2 + b2)
            ulp = np.maximum(np.abs(ref), 1e-30) * 2.0 ** -7 + acc * (1 + 2.0 ** -7)
            bad = np.abs(got - ref) > ulp
            out[name + "_ulp_flips"] = int((got != ref).sum())
            assert not bad.any(), (name, np.argwhere(bad)[:5])
        else:
            out[name + "_max_abs"] = float(np.abs(got - ref).max())
            assert out[name + "_max_abs"] < 1e-5
    return out
