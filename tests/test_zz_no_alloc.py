"""The allocation-free indexer entry point (dsa_indexer_topk_noalloc).

It serves callers that cannot give the library device memory on demand --
for example an inference engine whose allocator has already claimed all of
HBM for its KV-cache pool, or a plain C program with no allocator of its
own.  Its scratch is a fixed 72 MiB device array inside the library, shared
by every call.  These tests call it through the C ABI twice in a row, on two
different shapes, and require exactly the indices that the workspace-taking
entry point dsa_indexer_topk returns for the same inputs; a shape whose
scratch does not fit must be refused before anything runs.  This file is
collected last on purpose."""
import numpy as np
import pytest

from gpu_util import indexer_inputs_host, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_13_b200 import dsa as _dsa
    _dsa.lib()
    return _dsa


def _both(dsa, seed, B, Lq, Lk, start_pos, H, d, k, integer):
    q, kk, w = indexer_inputs_host(seed, B, Lq, Lk, H, d, integer=integer)
    qd, kd, wd = to_dev_bf16(q), to_dev_bf16(kk), to_dev_f32(w)
    want = dsa.indexer_topk(qd, kd, wd, k, start_pos=start_pos)
    got = dsa.indexer_topk_noalloc(qd, kd, wd, k, start_pos=start_pos)
    dsa.check_device_errors()
    return got.cpu().numpy(), want.cpu().numpy()


def test_noalloc_matches_workspace_entry_point_twice(dsa):
    # call 1: prefill-shaped rows (float inputs, ragged length, compactions)
    got, want = _both(dsa, 41, 1, 3000, 3000, 0, 64, 128, 512, integer=False)
    np.testing.assert_array_equal(got, want)
    # call 2 right after: decode-shaped rows whose key range is split across
    # CTAs and merged -- a different layout of the same shared scratch
    got, want = _both(dsa, 42, 4, 1, 30000, 30000, 64, 128, 2048, integer=True)
    np.testing.assert_array_equal(got, want)


def test_noalloc_refuses_shapes_beyond_its_scratch(dsa):
    import torch
    B, Lq, Lk, start_pos, H, d, k = 12, 12, 50000, 40000, 64, 128, 2048
    need = dsa.indexer_topk_workspace(B, Lq, Lk, start_pos, H, d, k)
    assert need > dsa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Lq, H, d), dtype=torch.bfloat16, device="cuda")
    kk = torch.zeros((B, Lk, d), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((B, Lq, H), dtype=torch.float32, device="cuda")
    with pytest.raises(dsa.DSAError) as e:
        dsa.indexer_topk_noalloc(q, kk, w, k, start_pos=start_pos)
    assert e.value.status == dsa.DSA_ERR_WORKSPACE
