"""The static-scratch variant of token-selective propagation.

kvc_tsp_select_gather_static serves callers that cannot allocate device
memory for a workspace (code that must keep away from the process' device
allocator).  Its scratch is an array compiled into the library, shared by
every call on a device, so two calls in a row must each give exactly what the
workspace variant kvc_tsp_select_gather gives on the same inputs: no state may
leak from the first call into the second.  This file sorts last so that a run
stopping at its first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_score_b200 import kvc, synth
from kv_cache_compression_score_b200.runner import TspSelector, from_device, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from kv_cache_compression_score_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _case(seed, S, w, n_rows, k_tsp, D):
    raw = torch.from_numpy(synth.random_scores(seed, (n_rows, S), n_levels=0)).cuda()
    hidden = to_device(synth.hidden_states(seed + 1, S, D, "bf16"), "bf16")
    return raw, hidden


def test_static_scratch_matches_workspace_variant_twice():
    w, pool_k = 32, 7
    # second call: shorter sequence and smaller selection than the first, so
    # stale scratch from the first call would show up in its result
    cases = [(91, 9000, 8, 1800, 256), (92, 4000, 4, 500, 512)]
    for seed, S, n_rows, k_tsp, D in cases:
        raw, hidden = _case(seed, S, w, n_rows, k_tsp, D)
        ref = TspSelector(S, w, pool_k, k_tsp, D, "bf16")
        idx_ref, hid_ref = ref.run(raw, hidden)
        idx = torch.empty(k_tsp + w, dtype=torch.int32, device="cuda")
        hid = torch.empty((k_tsp + w, D), dtype=torch.bfloat16, device="cuda")
        kvc.kvc_tsp_select_gather_static(raw, w, pool_k, k_tsp, hidden, idx, hid)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
        assert np.array_equal(from_device(hid), from_device(hid_ref))


def test_static_scratch_at_its_limit():
    """S - w exactly at the array's capacity (262,144 pooled prefix scores):
    the last element of the array is written and read; one more is refused."""
    w, pool_k, k_tsp, D = 32, 7, 300, 8
    S = 262144 + w
    raw, hidden = _case(93, S, w, 1, k_tsp, D)
    ref = TspSelector(S, w, pool_k, k_tsp, D, "bf16")
    idx_ref, hid_ref = ref.run(raw, hidden)
    idx = torch.empty(k_tsp + w, dtype=torch.int32, device="cuda")
    hid = torch.empty((k_tsp + w, D), dtype=torch.bfloat16, device="cuda")
    kvc.kvc_tsp_select_gather_static(raw, w, pool_k, k_tsp, hidden, idx, hid)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
    assert np.array_equal(from_device(hid), from_device(hid_ref))
    raw1 = torch.zeros((1, S + 1), dtype=torch.float32, device="cuda")
    hidden1 = torch.zeros((S + 1, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_tsp_select_gather_static(raw1, w, pool_k, k_tsp, hidden1, idx, hid)
    assert e.value.status == kvc.KVC_ERR_UNSUPPORTED


def test_static_scratch_rejects_oversize():
    S, w = 262144 + 64, 32
    raw = torch.zeros((1, S), dtype=torch.float32, device="cuda")
    hidden = torch.zeros((S, 8), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(64 + w, dtype=torch.int32, device="cuda")
    hid = torch.empty((64 + w, 8), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_tsp_select_gather_static(raw, w, 7, 64, hidden, idx, hid)
    assert e.value.status == 2 and "static-scratch" in str(e.value)
