"""NaN inputs in the oracle: the reading that NaN propagates through the
max-based scales to exactly the outputs that use them.

  Q NaN -> the rows of its quantisation block (per-token scales: its row);
  K NaN -> the K channel mean, every K scale, the whole head;
  V NaN -> the channel's scale, that output column of the whole head.
Exact float64 attention on the same input turns the same or fewer outputs
into NaN (a Q NaN there spoils only its own row).
"""

import numpy as np
import pytest

from oracle import attention as A
import workloads as W


def _inputs():
    w = W.custom(1, 2, 300, 32, seed=71)
    q, k, v = (t.float().numpy() for t in W.make_inputs(w))
    return q, k, v


@pytest.mark.parametrize("block_q,nan_rows", [(128, np.arange(128, 256)), (1, np.array([140]))])
def test_q_nan_spoils_the_rows_of_its_scale(block_q, nan_rows):
    q, k, v = _inputs()
    q[0, 0, 140, 3] = np.nan
    o = A.attn_quant_emul_i8f8(q, k, v, block_q=block_q, tau=4.0)
    bad = np.isnan(o[0]).any(axis=1)
    assert np.array_equal(np.nonzero(bad)[0], nan_rows)
    assert np.isnan(o[0][nan_rows]).all()
    assert np.isfinite(o[1]).all()                      # the other head
    assert np.isnan(A.attn_exact(q, k, v)[0][140]).all()


def test_k_nan_spoils_the_head():
    q, k, v = _inputs()
    k[0, 1, 7, 30] = np.nan
    o = A.attn_quant_emul_i8f8(q, k, v, tau=4.0)
    assert np.isnan(o[1]).all()
    assert np.isfinite(o[0]).all()


def test_v_nan_spoils_one_output_column():
    q, k, v = _inputs()
    v[0, 0, 250, 9] = np.nan
    o = A.attn_quant_emul_i8f8(q, k, v, tau=4.0)
    assert np.isnan(o[0][:, 9]).all()
    assert np.isfinite(np.delete(o[0], 9, axis=1)).all()
    assert np.isfinite(o[1]).all()
