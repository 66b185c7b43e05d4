"""The split-KV scheduler on the GPU against the oracle's specification, bit-exact.

The 512-thread scheduler gives each thread ceil(batch / 512) consecutive sequences; the cases
straddle those boundaries, with empty sequences, one-page and long sequences, and part counts
from 1 to more than the batch.
"""

import numpy as np
import pytest
import torch

from oracle import metadata as spec
from paged_mla_decode_11_b200 import ops

pytestmark = pytest.mark.gpu


def lengths(batch, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 5000, size=batch)
    lens[rng.random(batch) < 0.1] = 0          # empty sequences
    lens[rng.random(batch) < 0.05] = 64        # exactly one page
    if batch > 3:
        lens[batch // 3] = 70000               # one long sequence
    return lens.astype(np.int32)


@pytest.mark.parametrize("batch", [1, 2, 31, 32, 33, 95, 1000, 1023, 1024, 1025, 3000, 16384])
@pytest.mark.parametrize("rows", [16, 128])
def test_plan_matches_specification(batch, rows):
    for num_parts in (1, 7, 148, batch + 5):
        lens = lengths(batch, seed=batch * 7 + rows + num_parts)
        tile, splits = ops.get_mla_metadata(torch.from_numpy(lens).cuda(), rows, 1, num_parts=num_parts)
        torch.cuda.synchronize()
        want_tiles, want_splits = spec.schedule(lens.tolist(), num_parts, rows)
        assert tile.cpu().tolist() == want_tiles
        assert splits.cpu().tolist() == want_splits


@pytest.mark.parametrize("rows,h_kv", [(16, 1), (64, 1), (128, 1), (256, 1), (64, 2)])
def test_metadata_size_is_the_default_part_count(rows, h_kv):
    # the host-side sizing call and the scheduler's default agree on the current device
    lens = torch.from_numpy(lengths(40, seed=rows + h_kv)).cuda()
    tile, splits = ops.get_mla_metadata(lens, rows, h_kv)
    assert ops.metadata_size(40, rows, h_kv) == tile.shape[0]
    assert tile.shape[0] == ops.num_parts_for(ops.device_sm_count(), rows, h_kv)


@pytest.mark.parametrize("n_lists", [1, 33, 1000, 16384])
def test_csr_plan_matches_specification(n_lists):
    # the sparse decode's plan: the same specification over key-list lengths given as offsets
    counts = lengths(n_lists, seed=n_lists)
    row_ptr = np.zeros(n_lists + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    for rows, num_parts in ((16, 148), (8, 7)):
        tile, splits = ops.get_mla_metadata_csr(torch.from_numpy(row_ptr).cuda(), rows, 1, num_parts=num_parts)
        torch.cuda.synchronize()
        want_tiles, want_splits = spec.schedule(counts.tolist(), num_parts, rows)
        assert tile.cpu().tolist() == want_tiles
        assert splits.cpu().tolist() == want_splits
