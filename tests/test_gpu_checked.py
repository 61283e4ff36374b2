"""The bounds-checked build on the small parity cases.

``libbfa_checked.so`` is the library compiled with ``-DBFA_CHECKED``: every
plan-indexed access of the planner, forward and backward kernels checks its
bounds (an index outside its array is skipped and flagged, never trapped), and
every plan array is followed by guard bytes.  ``bfa_plan_device_status`` reports
either as ``BFA_ERR_BOUNDS``.  It stands in for a memory checker, which is not
available here.  This test runs a set of the small forward, backward and plan
parity tests in a subprocess that loads the checked build; the tests' conftest
then verifies every plan they create after each test.  They must all pass (the
outputs still match the oracle) with every plan's status clean, at the small
sizes and on the full-size workloads, the bench's causal 8192 launch included.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "mask_skipping_flashattention_b200", "libbfa_checked.so")

CASES = [
    "tests/test_gpu_plan.py::test_dense_plan_random",
    "tests/test_gpu_plan.py::test_blockid_plan_random_ragged",
    "tests/test_gpu_plan.py::test_varlen_plan_ragged_unequal",
    "tests/test_gpu_plan.py::test_bsr_plan_small",
    "tests/test_gpu_plan.py::test_general_block_sparse_plans",
    "tests/test_gpu_plan.py::test_predicate_plan_batched",
    "tests/test_gpu_plan.py::test_transposed_lists_dense",
    "tests/test_gpu_fwd.py::test_tiny_blockcausal",
    "tests/test_gpu_fwd.py::test_blockcausal_gqa_cross_columns",
    "tests/test_gpu_fwd.py::test_blockids_unsorted_and_sorted_key_tiles",
    "tests/test_gpu_fwd.py::test_varlen_small_all_rows",
    "tests/test_gpu_fwd.py::test_dense_ragged_gqa",
    "tests/test_gpu_fwd.py::test_all_true_and_empty_masks",
    "tests/test_gpu_fwd.py::test_general_block_sparse_forward",
    "tests/test_gpu_fwd.py::test_paged_kv_varlen",
    "tests/test_gpu_fwd.py::test_predicate_forward",
    "tests/test_gpu_fwd.py::test_block_skipping_drops_far_tiles",
    "tests/test_gpu_fwd.py::test_max_jump_in_a_later_key_tile",
    "tests/test_gpu_bwd.py::test_dense_random_masks",
    "tests/test_gpu_bwd.py::test_blockids_with_padding_and_cross_columns",
    "tests/test_gpu_bwd.py::test_positional_window_batched",
    "tests/test_gpu_bwd.py::test_predicate_terms",
    "tests/test_gpu_bwd.py::test_general_block_sparse_with_validity",
    "tests/test_gpu_bwd.py::test_varlen_causal_packed",
    "tests/test_gpu_bwd.py::test_fused_and_two_pass_forms_agree",
    "tests/test_gpu_bwd.py::test_two_pass_form_is_bitwise_reproducible",
    "tests/test_gpu_plan.py::test_bsr_packed_plans",
    "tests/test_gpu_fwd.py::test_bsr_packed_forward",
    "tests/test_gpu_bwd.py::test_bsr_packed_backward",
    # full-size workloads, the bench's own launch among them
    "tests/test_gpu_plan.py::test_dense_plan_causal_8192",
    "tests/test_gpu_plan.py::test_bsr_plan_workload_full_size_every_group",
    "tests/test_gpu_fwd.py::test_causal_8192_full_size_sampled",
    "tests/test_gpu_fwd.py::test_varlen_workload",
    "tests/test_gpu_fwd.py::test_bsr_workload_sampled",
    "tests/test_gpu_fwd.py::test_union_workload_sampled",
    "tests/test_gpu_bwd.py::test_bsr_workload_one_kv_group",
]


def test_checked_build_runs_the_small_parity_cases_clean():
    assert os.path.exists(CHECKED), "libbfa_checked.so is built with libbfa.so (build.py)"
    env = dict(os.environ, BFA_LIBRARY="checked")
    who = subprocess.run([sys.executable, "-c", "import mask_skipping_flashattention_b200 as b; "
                          "print(b.library_path); print(b._L.bfa_version().decode())"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert who.returncode == 0, who.stderr[-2000:]
    assert "libbfa_checked.so" in who.stdout and "checked" in who.stdout, who.stdout
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider", *CASES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout, r.stdout[-2000:]
