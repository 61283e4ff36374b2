"""Shared test utilities: oracle plans for each mask form and output comparison."""

from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oa
from oracle import masks as om
from oracle import plan as op

# Tolerances of the forward against the float64 oracle (bf16 N(0,1) inputs,
# fp32 accumulation): output max-abs 1e-2, LSE max-abs 1e-3, and -inf LSE
# positions identical.
O_ATOL = 1e-2
LSE_ATOL = 1e-3


def oracle_plan_for_groups(masks):
    return op.plan_masks([np.asarray(m, dtype=bool) for m in masks])


def assert_plan_equal(got, ref):
    """Bit-exact plan comparison: classes, lists, partial flags, fine words, order."""
    np.testing.assert_array_equal(got["row_ptr"], ref["row_ptr"], err_msg="row_ptr")
    np.testing.assert_array_equal(got["kv_tile"], ref["kv_tile"], err_msg="kv_tile")
    np.testing.assert_array_equal(got["partial"], ref["partial"], err_msg="partial flags")
    np.testing.assert_array_equal(got["order"], ref["order"], err_msg="order")
    ref_cls = np.concatenate([c.reshape(-1) for c in ref["cls"]]) if ref["cls"] else np.zeros(0, np.uint8)
    np.testing.assert_array_equal(got["classes"], ref_cls, err_msg="classes")
    if "fine" in got:
        np.testing.assert_array_equal(got["fine"], ref["fine"], err_msg="fine words")
    if "pair_row" in got:
        np.testing.assert_array_equal(got["pair_row"], ref["pair_row"], err_msg="pair rows")
        np.testing.assert_array_equal(got["pair_order"], ref["pair_order"], err_msg="pair order")


def compare_rows(O_gpu, L_gpu, O_ref, L_ref, where=""):
    """O_gpu (n, D) bf16/float tensor or array vs float64 oracle rows."""
    O_gpu = np.asarray(O_gpu.float().cpu() if isinstance(O_gpu, torch.Tensor) else O_gpu, dtype=np.float64)
    O_ref = np.asarray(O_ref, dtype=np.float64)
    assert np.all(np.isfinite(O_gpu)), f"non-finite output {where}"
    err = np.abs(O_gpu - O_ref).max() if O_ref.size else 0.0
    assert err <= O_ATOL, f"output max-abs {err:.3e} > {O_ATOL} {where}"
    if L_gpu is not None:
        L_gpu = np.asarray(L_gpu.cpu() if isinstance(L_gpu, torch.Tensor) else L_gpu, dtype=np.float64)
        inf_g, inf_r = np.isneginf(L_gpu), np.isneginf(L_ref)
        assert np.array_equal(inf_g, inf_r), f"-inf LSE positions differ {where}"
        fin = ~inf_r
        lerr = np.abs(L_gpu[fin] - L_ref[fin]).max() if fin.any() else 0.0
        assert lerr <= LSE_ATOL, f"LSE max-abs {lerr:.3e} > {LSE_ATOL} {where}"
        return err, lerr
    return err, 0.0


def check_bshd(out, lse, q, k, v, mask_for, scale, pairs, rows=None, where=""):
    """Compare (b, h) pairs of a batched forward with the oracle (optionally a row subset)."""
    Os, Ls = oa.attention_bshd(q, k, v, mask_for, scale, heads=pairs, rows=rows)
    worst = (0.0, 0.0)
    for (b, h) in pairs:
        og = out[b, :, h, :] if rows is None else out[b, rows, h, :]
        lg = None if lse is None else (lse[b, h] if rows is None else lse[b, h, rows])
        e = compare_rows(og, lg, Os[(b, h)], Ls[(b, h)], where=f"{where} (b={b}, h={h})")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    return worst


# Worst-case error of the bf16 path, used where the softmax is far peakier than
# the default scale makes it: P is rounded to bf16 before P V (relative error at
# most u = 2^-8 per weight, so at most u * max|v| on a weighted mean of v) and the
# output is rounded to bf16 (at most u * |O|); fp32 accumulation adds ~1e-5.
BF16_U = 2.0 ** -8


def peaked_bound(O_ref, vmax):
    return BF16_U * (np.abs(O_ref) + vmax) + 1e-4


def sample_rows(n, k, seed, must=()):
    rng = np.random.default_rng(seed)
    r = set(int(x) for x in rng.choice(n, size=min(k, n), replace=False))
    r.update(int(x) for x in must if 0 <= x < n)
    return np.array(sorted(r), dtype=np.int64)
