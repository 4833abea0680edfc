"""topk_select_noalloc: the context-free variant for callers that cannot
allocate device memory (engines that plan all memory up front, plugin hosts
without an allocator).  Its scratch is a static device array, so
this test checks, through the C ABI, that two calls in a row -- the second on
a different shape, after the first left its contents in the shared array --
give exactly what topk_select gives."""

import numpy as np
import pytest

from page_scoring_top_b200 import synth
from helpers import poisoned_outputs, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_noalloc_matches_topk_select_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from page_scoring_top_b200 import binding
    ctx = binding.Context(0, max_rows=32, max_n=65536, max_k=256)
    cases = [
        (synth.score_rows(4242, 8, 65536, "normal"), None, 256),              # many chunks per row
        (synth.score_rows(4243, 32, 20000, "levels16"),                        # ties, ragged
         np.array([20000, 19999, 1, 0] * 8, np.int32), 100),
    ]
    for s, lengths, K in cases:
        sd = to_dev(s)
        ln = None if lengths is None else to_dev(lengths)
        ref_i, ref_v = poisoned_outputs(s.shape[0], K)
        binding.topk_select(ctx, sd, ln, K, ref_i, ref_v)
        got_i, got_v = poisoned_outputs(s.shape[0], K)
        L = binding.lib()
        rc = L.topk_select_noalloc(sd.data_ptr(), None if ln is None else ln.data_ptr(), s.shape[0],
                                   s.shape[1], s.shape[1], K, got_i.data_ptr(), got_v.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
        assert rc == 0, binding.strerror(rc)
        torch.cuda.synchronize()
        assert torch.equal(got_i, ref_i)
        assert torch.equal(got_v.view(torch.int32), ref_v.view(torch.int32))
    # the Python wrapper runs the same call on the tensor's device
    s, K = synth.score_rows(4244, 3, 5000, "uniform"), 64
    sd = to_dev(s)
    ref_i, ref_v = poisoned_outputs(3, K)
    binding.topk_select(ctx, sd, None, K, ref_i, ref_v)
    got_i, got_v = poisoned_outputs(3, K)
    binding.topk_select_noalloc(sd, None, K, got_i, got_v)
    torch.cuda.synchronize()
    assert torch.equal(got_i, ref_i)
    assert torch.equal(got_v.view(torch.int32), ref_v.view(torch.int32))
    # beyond the scratch limit: a clear error, nothing launched
    # (256 rows x 4 chunks x K = 2048 candidates: 2M entries, twice the limit)
    big = torch.zeros((256, 65536), device="cuda")
    out = torch.empty((256, 2048), dtype=torch.int32, device="cuda")
    rc = binding.lib().topk_select_noalloc(big.data_ptr(), None, 256, 65536, 65536, 2048,
                                           out.data_ptr(), None, None)
    assert rc == binding.IDX_ENOWORKSPACE
    ctx.close()
