"""Pure-Python brute force of the hybrid layer, for tiny inputs only.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  It is written
independently of ``vnsa_oracle.c`` -- dictionaries keyed by token / block,
Python ``math`` only -- so that the C oracle can be checked against a second
implementation of the same definitions:

  * "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
    notes), section "Method": vision/text split, the three branches, the
    per-head sigmoid gate, dense GQA for text, outputs at original positions;
  * the readings R1-R10 and R13 (overlapping compression blocks) stated at
    the top of ``vnsa_oracle.c``.

The top-k step is not sorted here: every subset of the candidate blocks of the
right size is enumerated and the unique subset whose members all beat all
non-members under the strict order (importance descending, block index
ascending) is taken.  Exactly one subset has that property, which the code
asserts.
"""
from __future__ import annotations

import itertools
import math


def _dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def _softmax_attend(qv, keyvals, scale):
    """keyvals: dict key_id -> (k_vec, v_vec).  Returns (o, {key_id: p})."""
    if not keyvals:
        return [0.0] * len(qv), {}
    logits = {kid: scale * _dot(qv, kv[0]) for kid, kv in keyvals.items()}
    top = max(logits.values())
    weights = {kid: math.exp(s - top) for kid, s in logits.items()}
    total = sum(weights.values())
    probs = {kid: w / total for kid, w in weights.items()}
    o = [0.0] * len(qv)
    for kid, pr in probs.items():
        vv = keyvals[kid][1]
        for e in range(len(o)):
            o[e] += pr * vv[e]
    return o, probs


def _bf16(x):
    """Round to nearest bf16 (8 significant bits), ties to even, via frexp."""
    if x == 0.0 or not math.isfinite(x):
        return x
    m, e = math.frexp(x)             # x = m * 2**e, 0.5 <= |m| < 1
    e = max(e, -125)                 # keep bf16 subnormal spacing 2**-133
    scaled = x * 2.0 ** (8 - e)      # 8 significant bits above the point
    r = round(scaled)                # Python round(): half to even
    return r * 2.0 ** (e - 8)


def _topm(imp_by_block, candidates, m):
    """Unique m-subset of candidates beating all others (R5 order)."""
    def better(a, b):
        return (imp_by_block[a] > imp_by_block[b]) or (
            imp_by_block[a] == imp_by_block[b] and a < b)
    cands = sorted(candidates)
    if len(cands) <= m:
        return set(cands)
    winners = []
    for subset in itertools.combinations(cands, m):
        rest = [c for c in cands if c not in subset]
        if all(better(a, b) for a in subset for b in rest):
            winners.append(set(subset))
    assert len(winners) == 1, "strict order must give one top-m subset"
    return winners[0]


def layer(q, k, v, is_vision, gate, w_k, w_v, *, h_q, h_kv, d, block, top_k,
          window, force_first=True, force_local=True, scale=None,
          round_cmp_bf16=False, stride=None):
    """All rows of the layer.  Array-likes are nested lists / numpy arrays:
    q [n][h_q][d], k, v [n][h_kv][d], gate [n][h_q][3], w_k, w_v [d][d].
    ``stride``: compression stride (None: the block size).
    Returns dict(out=[n][h_q][d], idx={(t, g): sorted list}, imp={(t,g):{j:val}}
    (selection-block importance), o_cmp / o_slc / o_swa = {(t, h): vec})."""
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    n = len(is_vision)
    r = h_q // h_kv
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    # Partition by the modality flag: position -> vision rank.
    vision_rank = {}
    for t in range(n):
        if is_vision[t]:
            vision_rank[t] = len(vision_rank)
    pos_of_rank = {i: t for t, i in vision_rank.items()}
    nv = len(vision_rank)
    nb = nv // block
    stride = block if stride is None else stride
    # Compression blocks: the vision ranks each one averages (they overlap
    # when the stride is below the block size).
    cmp_members = {}
    c = 0
    while c * stride + block <= nv:
        cmp_members[c] = [c * stride + u for u in range(block)]
        c += 1
    # Compression keys/values per (block, kv head): mean over the block's
    # tokens, then the row vector times W.
    kcmp, vcmp = {}, {}
    for j, ranks in cmp_members.items():
        members = [pos_of_rank[u] for u in ranks]
        for g in range(h_kv):
            kbar = [sum(float(k[t][g][e]) for t in members) / block for e in range(d)]
            vbar = [sum(float(v[t][g][e]) for t in members) / block for e in range(d)]
            kc = [sum(kbar[e] * float(w_k[e][c]) for e in range(d)) for c in range(d)]
            vc = [sum(vbar[e] * float(w_v[e][c]) for e in range(d)) for c in range(d)]
            if round_cmp_bf16:
                kc = [_bf16(x) for x in kc]
                vc = [_bf16(x) for x in vc]
            kcmp[(j, g)] = kc
            vcmp[(j, g)] = vc
    out = [[[0.0] * d for _ in range(h_q)] for _ in range(n)]
    res = dict(out=out, idx={}, imp={}, o_cmp={}, o_slc={}, o_swa={})
    for t in range(n):
        if t not in vision_rank:
            for h in range(h_q):
                g = h // r
                kv = {u: ([float(x) for x in k[u][g]], [float(x) for x in v[u][g]])
                      for u in range(t + 1)}
                o, _ = _softmax_attend([float(x) for x in q[t][h]], kv, scale)
                out[t][h] = o
            continue
        i = vision_rank[t]
        visible = [j for j in range(nb) if (j + 1) * block - 1 <= i]
        cmp_visible = [cb for cb, ranks in cmp_members.items() if max(ranks) <= i]
        for g in range(h_kv):
            heads = [g * r + x for x in range(r)]
            imp_cmp = {cb: 0.0 for cb in cmp_visible}
            per_head_cmp = {}
            for h in heads:
                kv = {cb: (kcmp[(cb, g)], vcmp[(cb, g)]) for cb in cmp_visible}
                o, probs = _softmax_attend([float(x) for x in q[t][h]], kv, scale)
                per_head_cmp[h] = o
                for cb, pr in probs.items():
                    imp_cmp[cb] += pr
            # each compression block's mass goes to the selection blocks its
            # tokens fall in, one token's share (1 / block) at a time
            imp = {j: 0.0 for j in visible}
            for cb, mass in imp_cmp.items():
                for u in cmp_members[cb]:
                    if u // block in imp:
                        imp[u // block] += mass / block
            res["imp"][(t, g)] = imp
            forced = set()
            if force_first:
                forced.add(0)
            if force_local:
                forced.add(i // block)
            cands = [j for j in visible if j not in forced]
            chosen = forced | _topm(imp, cands, top_k - len(forced))
            res["idx"][(t, g)] = sorted(chosen)
            slc_tokens = [pos_of_rank[u] for u in range(nv)
                          if u // block in chosen and u <= i]
            swa_tokens = [pos_of_rank[u] for u in range(max(0, i - window + 1), i + 1)]
            for h in heads:
                qv = [float(x) for x in q[t][h]]
                kv_s = {u: ([float(x) for x in k[u][g]], [float(x) for x in v[u][g]])
                        for u in slc_tokens}
                kv_w = {u: ([float(x) for x in k[u][g]], [float(x) for x in v[u][g]])
                        for u in swa_tokens}
                o_s, _ = _softmax_attend(qv, kv_s, scale)
                o_w, _ = _softmax_attend(qv, kv_w, scale)
                o_c = per_head_cmp[h]
                gl = [float(x) for x in gate[t][h]]
                out[t][h] = [sig(gl[0]) * o_c[e] + sig(gl[1]) * o_s[e] + sig(gl[2]) * o_w[e]
                             for e in range(d)]
                res["o_cmp"][(t, h)] = o_c
                res["o_slc"][(t, h)] = o_s
                res["o_swa"][(t, h)] = o_w
    return res
