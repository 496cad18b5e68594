"""Host-side checks of the Python binding (no GPU): caller-supplied output
buffers and workspaces are checked against what the call writes before any
launch, and the data-parallel loss object drops outputs sized for another
step."""

from __future__ import annotations

import pytest
import torch

import lm_head_projection_b200 as pkg
from lm_head_projection_b200.dp import DataParallelFusedLinearLoss


def _inputs(BT=8, H=16, V=32, dt=torch.bfloat16):
    X = torch.zeros(BT, H, dtype=dt)
    W = torch.zeros(V, H, dtype=dt)
    b = torch.zeros(V, dtype=dt)
    Q = torch.zeros(BT, V, dtype=dt)
    return X, W, b, Q


@pytest.mark.parametrize("name,bad", [
    ("dX", lambda BT, H, V: torch.empty(BT - 1, H, dtype=torch.bfloat16)),
    ("dX", lambda BT, H, V: torch.empty(BT, H, dtype=torch.float32)),
    ("dW", lambda BT, H, V: torch.empty(V, H, dtype=torch.bfloat16)),  # accum_fp32: fp32
    ("dW", lambda BT, H, V: torch.empty(V // 2, H, dtype=torch.float32)),
    ("db", lambda BT, H, V: torch.empty(V + 1, dtype=torch.float32)),
    ("loss", lambda BT, H, V: torch.empty(1, dtype=torch.float32)),
    ("dX", lambda BT, H, V: torch.empty(H, BT, dtype=torch.bfloat16).t()),  # not contiguous
])
def test_wrong_output_buffers_are_refused_before_any_launch(name, bad):
    X, W, b, Q = _inputs()
    BT, H = X.shape
    V = W.shape[0]
    with pytest.raises(ValueError, match=name):
        pkg.forward_backward(X, W, b, Q, compute_dW=True, compute_db=True, accum_fp32=True,
                             out={name: bad(BT, H, V)})
    with pytest.raises(ValueError, match=name):
        pkg.cross_entropy_forward_backward(X, W, b, torch.zeros(BT, dtype=torch.int64),
                                           compute_dW=True, compute_db=True, accum_fp32=True,
                                           out={name: bad(BT, H, V)})


def test_workspace_of_another_dtype_is_refused():
    X, W, b, Q = _inputs()
    with pytest.raises(ValueError, match="workspace"):
        pkg.forward_backward(X, W, b, Q, workspace=torch.empty(1 << 20, dtype=torch.float32))


def test_dp_loss_keeps_outputs_only_while_shapes_and_flags_stay():
    loss = DataParallelFusedLinearLoss("kl")
    X, W, b, _ = _inputs(BT=96)
    assert loss._reusable_out(X, W, b, True, True) is None
    loss.out = {"dX": torch.empty(96, 16)}
    assert loss._reusable_out(X, W, b, True, True) is loss.out
    X64 = torch.zeros(64, 16, dtype=torch.bfloat16)
    assert loss._reusable_out(X64, W, b, True, True) is None  # shorter batch
    loss.out = {"dX": torch.empty(64, 16)}
    assert loss._reusable_out(X64, W, b, False, True) is None  # frozen head now
    loss.out = {"dX": torch.empty(64, 16)}
    assert loss._reusable_out(X64, W, None, False, True) is None  # no bias: no db
