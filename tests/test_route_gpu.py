"""Routing prologue on the GPU against the oracle: bit-exact counts, offsets,
stable permutation and tile list."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
import oracle
from workloads.gen import distinct_uniform_ids, zipf_ids

pytestmark = pytest.mark.gpu


def _case(kind, rng):
    if kind == "uniform":
        return distinct_uniform_ids(rng, 4096, 8, 128), 128
    if kind == "zipf":
        return zipf_ids(rng, 8192, 8, 256, 1.1), 256
    if kind == "one_expert":
        return np.full((1000, 1), 7, np.uint32), 16
    if kind == "bad_ids":
        ids = rng.integers(0, 40, size=(700, 3)).astype(np.uint32)
        ids[5, 1] = 0xFFFFFFFF
        return ids, 32
    if kind == "single":
        return np.array([[3]], np.uint32), 8
    if kind == "many_experts":
        return rng.integers(0, 1024, size=(3000, 4)).astype(np.uint32), 1024
    if kind == "ragged_chunk":
        return rng.integers(0, 5, size=(4097, 1)).astype(np.uint32), 5
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["uniform", "zipf", "one_expert", "bad_ids", "single",
                                  "many_experts", "ragged_chunk"])
@pytest.mark.parametrize("tile_rows", [64, 256, 1])
def test_route_bit_exact(kind, tile_rows):
    rng = np.random.default_rng(21)
    ids, E = _case(kind, rng)
    ref_counts, ref_offsets, ref_sp, ref_tiles = oracle.route(ids, E, tile_rows)
    dev_ids = torch.from_numpy(np.ascontiguousarray(ids).view(np.int32)).cuda()
    ws = M.new_workspace(ids.shape[0], ids.shape[1], E)
    counts, offsets, sp, tiles = M.route(dev_ids, E, tile_rows, workspace=ws)
    torch.cuda.synchronize()
    u = lambda t: t.cpu().numpy().view(np.uint32)  # noqa: E731
    np.testing.assert_array_equal(u(counts), ref_counts)
    np.testing.assert_array_equal(u(offsets), ref_offsets)
    np.testing.assert_array_equal(u(sp), ref_sp)
    np.testing.assert_array_equal(u(tiles), ref_tiles)
    status = M.poll_error(ws)
    assert status == (5 if kind == "bad_ids" else 0)


def test_route_deterministic_reruns():
    rng = np.random.default_rng(22)
    ids = zipf_ids(rng, 8192, 8, 256, 1.1)
    dev_ids = torch.from_numpy(ids.view(np.int32)).cuda()
    a = M.route(dev_ids, 256, 256)
    b = M.route(dev_ids, 256, 256)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
