"""Shared test helpers: device upload of the seeded inputs and the parity checks."""

from __future__ import annotations

import numpy as np

import oracle

POISON_I32 = np.int32(np.uint32(0xA5A5A5A5).view(np.int32))


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def to_dev(arr):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr)).cuda()


def poisoned_outputs(rows, K):
    """idx/val outputs pre-filled with the 0xa5 pattern, so unwritten slots show."""
    import torch
    idx = torch.full((rows, K), int(POISON_I32), dtype=torch.int32, device="cuda")
    val = torch.full((rows, K), 0, dtype=torch.int32, device="cuda")
    val.fill_(int(POISON_I32))
    return idx, val.view(torch.float32)


def check_select_bit_exact(scores_f32, lengths_per_row, K, idx_gpu, val_gpu):
    """GPU indices equal the oracle's select on the same fp32 rows, element for
    element; values are bit-equal to the scores at those indices."""
    want_idx, want_val = oracle.topk_rows(scores_f32, K, lengths_per_row)
    bad = np.argwhere(idx_gpu != want_idx)
    assert bad.size == 0, "index mismatch at %s: gpu %s oracle %s" % (
        bad[:5].tolist(), idx_gpu[tuple(bad[0])], want_idx[tuple(bad[0])])
    if val_gpu is not None:
        assert np.array_equal(val_gpu.view(np.uint32), want_val.view(np.uint32)), "value bits differ"


def check_recall(idx_gpu, S_exact, lengths_per_row, K, floor=0.999):
    """recall@floor(3K/4) and recall@K against the oracle's own (double) top-K."""
    want, _ = oracle.topk_rows(S_exact, K, lengths_per_row)
    out = {}
    for m in (3 * K // 4, K):
        r = [oracle.recall(idx_gpu[i], want[i], m) for i in range(idx_gpu.shape[0])]
        out[m] = float(np.mean(r))
        assert out[m] >= floor, "recall@%d = %.5f" % (m, out[m])
    return out
