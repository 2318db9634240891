"""moe_permute on the GPU against the oracle: offsets, perm and inv byte-equal, for the
route classes of "MTP1 isolated gather/shared-add closure" (same, disjoint, overlap,
duplicate-free random) plus empty experts, one expert taking every token, M = 0, and
out-of-range ids reported through the device error word."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_35_b200.moe as moe

pytestmark = pytest.mark.gpu


def _routes(kind, M, K, E, rng):
    if kind == "same":
        row = rng.permutation(E)[:K]
        return np.tile(row, (M, 1))
    if kind == "disjoint":
        assert M * K <= E
        return rng.permutation(E)[:M * K].reshape(M, K)
    if kind == "overlap":
        pool = rng.permutation(E)[:K + 2]
        return np.stack([rng.permutation(pool)[:K] for _ in range(M)])
    if kind == "skewed":  # most tokens on the first few experts, many experts empty
        p = 1.0 / np.arange(1, E + 1) ** 1.5
        return np.stack([rng.choice(E, K, replace=False, p=p / p.sum()) for _ in range(M)])
    return np.stack([rng.permutation(E)[:K] for _ in range(M)])


@pytest.mark.parametrize("kind,M,K,E", [
    ("same", 37, 4, 16), ("disjoint", 16, 8, 256), ("overlap", 300, 6, 128), ("random", 1, 1, 1),
    ("random", 1, 10, 512), ("random", 4096, 8, 256), ("random", 8192, 8, 256), ("skewed", 2048, 10, 512),
    ("random", 333, 32, 1024), ("random", 65, 1, 8)])
def test_permute_matches_oracle(kind, M, K, E):
    rng = np.random.default_rng(M * 7 + K * 3 + E)
    ids = _routes(kind, M, K, E, rng).astype(np.int32)
    ro, rp, ri = oracle.permute(ids, E)
    for _ in range(2):  # deterministic: two runs byte-equal to the oracle
        off, perm, inv = moe.permute(torch.from_numpy(ids).cuda(), E)
        assert off.cpu().numpy().tobytes() == ro.tobytes()
        assert perm.cpu().numpy().tobytes() == rp.tobytes()
        assert inv.cpu().numpy().tobytes() == ri.tobytes()


def test_permute_one_expert_takes_all():
    M, K, E = 1000, 1, 64
    ids = np.full((M, K), 5, np.int32)
    off, perm, inv = moe.permute(torch.from_numpy(ids).cuda(), E)
    off = off.cpu().numpy()
    assert off[5] == 0 and off[6] == M and off[-1] == M
    np.testing.assert_array_equal(perm.cpu().numpy(), np.arange(M))


def test_permute_empty():
    ids = torch.empty((0, 4), dtype=torch.int32, device="cuda")
    off, perm, inv = moe.permute(ids, 16)  # M == 0: nothing is launched
    assert perm.numel() == 0


def test_permute_bad_ids_set_error_word():
    ids = torch.tensor([[0, 3], [1, 99], [-2, 2]], dtype=torch.int32, device="cuda")
    ws = torch.zeros(moe.permute_workspace_size(3, 2, 8), dtype=torch.uint8, device="cuda")
    off, perm, inv = moe.permute(ids, 8, ws)
    code = moe.get_error(ws)
    assert code & moe.DEVERR_BAD_EXPERT_ID
    assert moe.get_error(ws) == 0  # cleared by the read
    good = torch.tensor([[0, 3], [1, 2]], dtype=torch.int32, device="cuda")
    moe.permute(good, 8, ws)
    assert moe.get_error(ws) == 0
