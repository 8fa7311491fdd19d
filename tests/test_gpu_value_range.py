"""Values far outside the unit range.  bf16 inputs reach 3.4e38; the P V products
take fp16 operands, which stop at 65,504, so the layer hands V and V_cmp to them
divided by a power of two chosen from their largest magnitude in each call
(and multiplies it back).

V of a bf16 layer is scaled by 2^17 (131,072, beyond fp16's range) and by 2^-20
(about 1e-6, below fp16's normal range).  A power of two moves every value and
every rounding boundary together, so:
  * the scaled layer must equal the unscaled layer times the scale, bit for bit
    (V_cmp, the fp32 partial and the bf16 output all scale exactly);
  * in units of the scale its error against the fp64 oracle must stay within
    the unscaled workload's 2e-2.
"""
import numpy as np
import pytest

import oracle
from parity_util import check_selection, oracle_params, run_gpu
from sparse_attention_long_block_b200.inputs import Workload, generate

pytestmark = pytest.mark.gpu


def test_v_scaled_by_powers_of_two_far_from_unit_range():
    wl = Workload(name="vrange", n_vision=2048, n_text=96, top_k=8, window=128, seed=51)
    x = generate(wl)
    base = run_gpu(wl, x, want=("idx",))
    assert base["status"] == 0
    nv = wl.n_vision
    for scale in (2.0 ** 17, 2.0 ** -20):
        xs = dict(x)
        xs["v"] = (x["v"].astype(np.float64) * scale).astype(np.float32)  # exact
        g = run_gpu(wl, xs, want=("idx", "imp"))
        assert g["status"] == 0
        assert np.isfinite(g["out"]).all()
        # V does not enter the selection, and every step scales exactly
        assert np.array_equal(g["idx"], base["idx"])
        assert np.array_equal(g["out"].astype(np.float64), base["out"].astype(np.float64) * scale)
        o = oracle.forward(oracle_params(wl), xs["q"], xs["k"], xs["v"], xs["is_vision"],
                           xs["gate"], xs["w_k"], xs["w_v"], want=("idx", "imp"))
        gsel = np.transpose(g["idx"][:, :nv], (1, 0, 2))
        swapped = check_selection(gsel, o["idx"][:nv], o["imp"][:nv], wl.top_k,
                                  block=wl.block, ranks=np.arange(nv))
        ref = o["out"].copy()
        if swapped:  # near-tied blocks the kernel chose: the oracle on its selection
            rows = np.nonzero(xs["is_vision"])[0][swapped].astype(np.int32)
            o2 = oracle.forward(oracle_params(wl), xs["q"], xs["k"], xs["v"], xs["is_vision"],
                                xs["gate"], xs["w_k"], xs["w_v"], rows=rows,
                                forced_idx=gsel[swapped])
            ref[rows] = o2["out"]
        err = float(np.abs(g["out"] - ref).max()) / scale
        assert err <= 2e-2, (scale, err)
