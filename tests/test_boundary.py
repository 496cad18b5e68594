"""C-ABI boundary tests that need no GPU: the library loads, exports every
symbol the header declares, sizes its workspace without any BT x V term, and
rejects bad arguments on the host before launching anything.

The argument-rejection tests pass placeholder pointer values that must never
reach a kernel, so they only run where no GPU is visible.
"""

import ctypes
import os
import re

import pytest
import torch

import lm_head_projection_b200 as pkg
from lm_head_projection_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flkl.h")

OK, INVALID, UNSUPPORTED, CUDA, TIMEOUT, WORKSPACE = range(6)


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"FLKL_API\s+[\w\s\*]*?\b(flkl_\w+)\s*\(", text)


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 7
    lib = ctypes.CDLL(pkg.library_path())
    for s in syms:
        assert hasattr(lib, s), s


def test_abi_version_and_status_strings():
    assert pkg.flkl_abi_version() == 1
    for s in range(6):
        assert pkg.flkl_status_string(s)
    assert "unknown" in pkg.flkl_status_string(99)


def test_workspace_size_rules():
    ws = pkg.flkl_workspace_size
    assert ws(-1, 64, 64, 1, 1, 0) == 0
    assert ws(4, 0, 64, 1, 1, 0) == 0
    assert ws(4, 64, 0, 1, 1, 0) == 0
    assert ws(4, 64, 64, 7, 1, 0) == 0
    assert ws(0, 64, 64, 1, 1, 0) > 0
    assert ws(4, 64, 64, 1, 1, 1) > ws(4, 64, 64, 1, 1, 0)
    assert ws(4, 64, 64, 1, 1, 0) % 256 == 0


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workspace_has_no_bt_by_v_buffer(name):
    """The two staged gradient blocks are at most BT x V/6 each (plus tile
    rounding), and of the logits only the first chunk's are kept (fp32, at
    most 256 MiB): the whole workspace stays below one BT x V array of the
    input dtype (the logits alone in fp32 would take two)."""
    w = WORKLOADS[name]
    elem = 4 if w.dtype == "fp32" else 2
    need = pkg.flkl_workspace_size(w.BT, w.H, w.V, 0 if w.dtype == "fp32" else 1, w.compute_dW,
                                   w.compute_db)
    full = w.BT * w.V * elem
    if w.V >= 8 * 256:
        assert need < full, (need, full)
        if w.dtype == "bf16":
            bounds = pkg.flkl_vocab_chunks(w.BT, w.H, w.V, 1, w.compute_dW, w.compute_db)
            assert max(b - a for a, b in zip(bounds, bounds[1:])) <= -(-w.V // 6) + 255
            rows32 = -(-w.BT // 32) * 32
            cols = min(bounds[1], (256 << 20) // (rows32 * 4) // 256 * 256)
            assert rows32 * cols * 4 <= 256 << 20


no_gpu = pytest.mark.skipif(torch.cuda.is_available(),
                            reason="placeholder pointers must not reach a real device")

P = 4096  # placeholder, 16-byte aligned, never dereferenced


def call(**kw):
    a = dict(X=P, W=P, b=None, Q=P, shift_labels=None, ignore_index=-100, BT=64, H=64, V=64,
             dtype=1, temperature=1.0, eps=1e-10, reduction=0, compute_dW=1, compute_db=0,
             accum_fp32=1, loss=P, dX=P, dW=P, db=None, workspace=P, workspace_bytes=0,
             stream=None)
    a.update(kw)
    return pkg.flkl_forward_backward(**a)


@no_gpu
@pytest.mark.parametrize("kw,expect", [
    (dict(reduction=3), UNSUPPORTED),           # reduction none refused
    (dict(reduction=7), INVALID),
    (dict(dtype=5), INVALID),
    (dict(temperature=0.0), INVALID),
    (dict(temperature=-1.0), INVALID),
    (dict(temperature=float("nan")), INVALID),
    (dict(temperature=float("inf")), INVALID),
    (dict(eps=-1e-3), INVALID),
    (dict(eps=float("nan")), INVALID),
    (dict(BT=-1), INVALID),
    (dict(H=0), INVALID),
    (dict(V=0), INVALID),
    (dict(H=60), UNSUPPORTED),                  # bf16 rows must be 16-byte multiples
    (dict(V=1004), UNSUPPORTED),
    (dict(dtype=0, H=62), UNSUPPORTED),
    (dict(BT=1 << 31), UNSUPPORTED),
    (dict(W=None), INVALID),
    (dict(X=None), INVALID),
    (dict(Q=None), INVALID),
    (dict(loss=None), INVALID),
    (dict(dX=None), INVALID),
    (dict(dW=None), INVALID),                   # compute_dW without dW
    (dict(compute_dW=0), INVALID),              # dW given while frozen
    (dict(compute_db=1, db=P), INVALID),        # db without bias
    (dict(compute_db=1, b=P), INVALID),         # db pointer missing
    (dict(compute_db=0, b=P, db=P), INVALID),   # db given but not asked for
    (dict(X=P + 8), UNSUPPORTED),               # misaligned
    (dict(Q=P + 4), UNSUPPORTED),
    (dict(dX=P + 2), UNSUPPORTED),
    (dict(shift_labels=P + 4), UNSUPPORTED),
    (dict(workspace=None), WORKSPACE),
    (dict(workspace=P + 16, workspace_bytes=1 << 40), WORKSPACE),  # not 256-aligned
    (dict(workspace_bytes=100), WORKSPACE),     # too small
])
def test_host_rejects_bad_arguments(kw, expect):
    assert call(**kw) == expect


@no_gpu
def test_empty_rows_allow_null_row_tensors_but_need_workspace():
    assert call(BT=0, X=None, Q=None, dX=None, workspace_bytes=0) == WORKSPACE


def test_python_module_refuses_reduction_none():
    with pytest.raises(ValueError):
        pkg.FusedLinearKLDivLoss(reduction="none")


@no_gpu
def test_ce_entry_needs_targets():
    assert pkg.flkl_ce_forward_backward(P, P, None, None, -100, 64, 64, 64, 1, 1.0, 0, 1, 0, 1,
                                        P, P, P, None, P, 0, None) == INVALID
    assert pkg.flkl_ce_forward_backward(P, P, None, P, -100, 64, 64, 64, 1, 1.0, 3, 1, 0, 1,
                                        P, P, P, None, P, 0, None) == UNSUPPORTED


def norm_call(layer=False, **kw):
    a = dict(dY=P, X=P, W=P, rows=64, H=4096, dtype=1, eps=1e-6, compute_dW=1, compute_db=0,
             accum_fp32=1, dX=P, dW=P, db=None, workspace=P, workspace_bytes=1 << 30,
             stream=None)
    a.update(kw)
    if layer:
        return pkg.flkl_layer_norm_backward(**a)
    a.pop("compute_db"), a.pop("db")
    return pkg.flkl_rms_norm_backward(**a)


def test_norm_workspace_size_rules():
    # one fp32 partial row per block and per gradient asked for; nothing when frozen
    assert pkg.flkl_norm_workspace_size(8192, 4096, 0, 0) == 0
    one = pkg.flkl_norm_workspace_size(8192, 4096, 1, 0)
    assert one == pkg.flkl_norm_workspace_size(8192, 4096, 0, 1) > 0
    assert pkg.flkl_norm_workspace_size(8192, 4096, 1, 1) == 2 * one
    # one fp32 row per CTA, at least 8 rows per CTA, at most 16 CTAs per SM
    assert one % 256 == 0 and one <= 8192 // 8 * 4096 * 4
    big = pkg.flkl_norm_workspace_size(1 << 22, 4096, 1, 0)
    assert big == pkg.flkl_norm_workspace_size(1 << 23, 4096, 1, 0) <= 148 * 16 * 4096 * 4
    assert pkg.flkl_norm_workspace_size(3, 64, 1, 0) == 256   # 3 rows -> 1 CTA
    assert pkg.flkl_norm_workspace_size(10, 8200, 1, 0) == 0  # H above the limit


@no_gpu
@pytest.mark.parametrize("layer", [False, True])
@pytest.mark.parametrize("kw,expect", [
    (dict(dtype=4), INVALID),
    (dict(rows=-1), INVALID),
    (dict(H=0), INVALID),
    (dict(eps=-1.0), INVALID),
    (dict(eps=float("nan")), INVALID),
    (dict(H=4100), UNSUPPORTED),                # not a multiple of 8
    (dict(H=8200), UNSUPPORTED),                # above 8192
    (dict(W=None), INVALID),
    (dict(X=None), INVALID),
    (dict(dY=None), INVALID),
    (dict(dX=None), INVALID),
    (dict(dW=None), INVALID),                   # compute_dW without dW
    (dict(compute_dW=0), INVALID),              # dW given while frozen
    (dict(X=P + 8), UNSUPPORTED),
    (dict(dW=P + 4), UNSUPPORTED),
    (dict(workspace=None), WORKSPACE),
    (dict(workspace=P + 16), WORKSPACE),        # not 256-aligned
    (dict(workspace_bytes=100), WORKSPACE),
])
def test_norm_host_rejects_bad_arguments(layer, kw, expect):
    assert norm_call(layer, **kw) == expect


@no_gpu
def test_layer_norm_bias_flag_needs_pointer():
    assert norm_call(True, compute_db=1) == INVALID            # db missing
    assert norm_call(True, compute_db=0, db=P) == INVALID      # db not asked for


@no_gpu
def test_selective_logprob_entries_check_their_arguments():
    fwd = lambda **kw: pkg.flkl_selective_logprob_forward(**{**dict(
        X=P, W=P, b=None, target=P, ignore_index=-100, BT=64, H=64, V=64, dtype=1,
        temperature=1.0, compute_dW=1, compute_db=0, logp=P, workspace=P,
        workspace_bytes=1 << 30, stream=None), **kw})
    bwd = lambda **kw: pkg.flkl_selective_logprob_backward(**{**dict(
        X=P, W=P, b=None, target=P, ignore_index=-100, BT=64, H=64, V=64, dtype=1,
        temperature=1.0, dlogp=P, compute_dW=1, compute_db=0, accum_fp32=1, dX=P, dW=P,
        db=None, workspace=P, workspace_bytes=1 << 30, stream=None), **kw})
    assert fwd(target=None) == INVALID
    assert fwd(logp=None) == INVALID
    assert fwd(logp=P + 2) == UNSUPPORTED
    assert fwd(temperature=0.0) == INVALID
    assert fwd(workspace_bytes=16) == WORKSPACE
    assert fwd(compute_db=1) == INVALID          # db needs a bias
    assert bwd(dlogp=None) == INVALID
    assert bwd(target=None) == INVALID
    assert bwd(dX=None) == INVALID
    assert bwd(dW=None) == INVALID               # compute_dW without dW
    assert bwd(H=60) == UNSUPPORTED


@no_gpu
def test_jsd_entry_checks_its_arguments():
    def jsd(**kw):
        a = dict(X=P, W=P, b=None, Xt=P, Wt=P, bt=None, shift_labels=None, ignore_index=-100,
                 BT=64, H=64, Ht=32, V=64, dtype=1, temperature=1.0, beta=0.5, reduction=0,
                 compute_dW=1, compute_db=0, accum_fp32=1, loss=P, dX=P, dW=P, db=None,
                 workspace=P, workspace_bytes=1 << 30, stream=None)
        a.update(kw)
        return pkg.flkl_jsd_forward_backward(**a)
    assert jsd(beta=0.0) == INVALID
    assert jsd(beta=1.0) == INVALID
    assert jsd(beta=float("nan")) == INVALID
    assert jsd(reduction=3) == UNSUPPORTED
    assert jsd(Xt=None) == INVALID
    assert jsd(Wt=None) == INVALID
    assert jsd(Ht=36) == UNSUPPORTED          # bf16 teacher rows: multiple of 8
    assert jsd(bt=P + 8) == UNSUPPORTED
    assert jsd(compute_db=1, db=P) == INVALID  # db needs a bias
    assert jsd(workspace_bytes=100) == WORKSPACE
    need = pkg.flkl_jsd_workspace_size(1024, 4096, 4096, 128256, 1, 1, 0)
    assert 0 < need < 1024 * 128256 * 2   # below one BT x V bf16 array


def test_launch_kind_names_follow_the_header_enum():
    """The binding's names of the profiled launch kinds are the header's
    flkl_launch_kind values, in order."""
    import os
    import re

    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "flkl.h")).read()
    body = hdr[hdr.index("typedef enum {\n  FLKL_LAUNCH_PREPARE"):hdr.index("} flkl_launch_kind;")]
    vals = {int(v): n for n, v in re.findall(r"FLKL_LAUNCH_(\w+)\s*=\s*(\d+)", body)}
    assert sorted(vals) == list(range(len(vals)))
    names = [vals[i].lower() for i in range(len(vals))]
    assert [n.replace("_", "") for n in names] == [k.replace("_", "").lower()
                                                   for k in pkg.LAUNCH_KINDS]
