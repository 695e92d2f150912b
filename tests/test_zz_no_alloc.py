"""moe_permute_static_ws: the permutation for callers that cannot allocate.

Some users of this library are handed only the tensors of a call and may not
allocate device memory while it runs (an inference engine's plugin execute
hook with a fixed memory pool, for example).  For them the library offers a
permutation whose scratch lives in a static array inside the library.  These
tests call it through the C ABI twice in a row, with different shapes, and
require exactly the output of the workspace-taking moe_permute (integer maps
and copied rows, so the tolerance is bit-exactness).

This file runs last so that a failure here comes after every other test has run.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import moe_layer_forward_b200 as m

    return m


def _buffers(T, E, k, d, dtype):
    return (torch.empty(E, dtype=torch.int32, device=DEV), torch.empty(E + 1, dtype=torch.int32, device=DEV),
            torch.empty(T * k, dtype=torch.int32, device=DEV), torch.empty((T, k), dtype=torch.int32, device=DEV),
            torch.empty((T * k, d), dtype=dtype, device=DEV))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_permute_matches_workspace_permute_twice(moe, dtype):
    # two calls in a row with different sizes: the second must not see the first's leftovers
    # the last case is the documented maximum: 65536 tokens and 256 experts fill all 256 x 256 counters
    for (T, E, k, d, seed) in [(1000, 64, 8, 128, 1), (300, 256, 8, 64, 2), (65536, 256, 8, 8, 3)]:
        idx = synth.distinct_topk(T, E, k, seed).to(DEV)
        v = synth.normal((T, d), seed, 1, dtype=dtype).to(DEV)
        ref = _buffers(T, E, k, d, dtype)
        got = _buffers(T, E, k, d, dtype)
        st_ref = torch.zeros(1, dtype=torch.int32, device=DEV)
        st_got = torch.zeros(1, dtype=torch.int32, device=DEV)
        moe.moe_permute(v, idx, E, *ref, dev_status=st_ref)
        moe.moe_permute_static_ws(v, idx, E, *got, dev_status=st_got)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        assert st_got.item() == st_ref.item() == 0


def test_static_scratch_permute_rejects_more_tokens_than_its_scratch_holds(moe):
    T, E, k, d = 65537, 16, 1, 8
    v = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((T, k), dtype=torch.int32, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_permute_static_ws(v, idx, E, *_buffers(T, E, k, d, torch.bfloat16))
    assert ei.value.status == 2  # MOE_ERR_UNSUPPORTED
