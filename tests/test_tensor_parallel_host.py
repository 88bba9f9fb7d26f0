"""Tensor-parallel TTQ on the host: two gloo ranks on the CPU run the
row- and column-parallel projections of tensor_parallel.py with a stand-in
for the CUDA calls built on the oracle, and rank 0 compares the result with
the oracle's unsplit layer. This checks the split, the collectives and the
assembly; the kernels behind the calls have their own parity tests."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """The calls tensor_parallel.py makes, computed by the oracle on CPU
    tensors (test double of the CUDA binding)."""

    def act_stats(self, X, p=2.0):
        import oracle
        return torch.from_numpy(oracle.act_sums(X.float().numpy(), p).astype(
            np.float32))

    def channel_moment_total(self, sums, T):
        return torch.tensor([np.sum(sums.double().numpy() / T)],
                            dtype=torch.float64)

    def awq_scales_sharded(self, sums, T, K_total, total, alpha, lam, p):
        import oracle
        s, inv = oracle.awq_scales_given_mean(
            sums.double().numpy(), T, float(total.item()) / K_total, alpha,
            lam, p)
        return (torch.from_numpy(s.astype(np.float32)),
                torch.from_numpy(inv.astype(np.float32)))

    def awq_scales(self, sums, T, alpha, lam, p):
        import oracle
        s, inv = oracle.awq_scales(sums.double().numpy(), T, alpha, lam, p)
        return (torch.from_numpy(s.astype(np.float32)),
                torch.from_numpy(inv.astype(np.float32)))

    def quantize_rtn_grouped(self, W, s, bits, group):
        import oracle
        return oracle.quantize(W.float().numpy(), s.numpy(), bits, group)

    def w_lowbit_gemm(self, X, inv, c, d, z, N, bits, group,
                      out_dtype=torch.bfloat16):
        import oracle
        Y = oracle.lowbit_gemm(X.float().numpy(), inv.numpy(), c, d, z, N,
                               bits, group)
        return torch.from_numpy(Y).to(out_dtype)


T, N, K, BITS, GROUP = 24, 40, 256, 4, 64


def _inputs():
    from test_weight_quantization_b200.inputs import activations, weights
    X = torch.from_numpy(activations(T, K, 5, "student_t", 0.05, 0, 20.0))
    W = torch.from_numpy(weights(N, K, 6))
    return X.to(torch.bfloat16).float(), W.to(torch.bfloat16).float()


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from test_weight_quantization_b200 import tensor_parallel as tp
    from test_weight_quantization_b200.ttq import TTQParams
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, W = _inputs()
        prm = TTQParams(bits=BITS, group=GROUP)
        k0, k1 = tp.shard_channels(K, world, GROUP)[rank]
        row = tp.RowParallelTTQLinear(W[:, k0:k1], K, prm, ops=OracleOps())
        out[f"row{rank}"] = row(X[:, k0:k1], out_dtype=torch.float32).numpy()
        n0, n1 = tp.shard_rows(N, world)[rank]
        col = tp.ColumnParallelTTQLinear(W[n0:n1], prm, ops=OracleOps())
        out[f"col{rank}"] = col(X, gather=True,
                                out_dtype=torch.float64).numpy()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def two_ranks():
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    return dict(out)


def _unsplit():
    import oracle
    X, W = _inputs()
    sums = oracle.act_sums(X.numpy())
    s, inv = oracle.awq_scales(sums.astype(np.float32).astype(np.float64), T,
                               0.5, 0.1, 2.0)
    s32, inv32 = s.astype(np.float32), inv.astype(np.float32)
    c, d, z = oracle.quantize(W.numpy(), s32, BITS, GROUP)
    return oracle.lowbit_gemm(X.numpy(), inv32, c, d, z, N, BITS, GROUP)


def test_row_parallel_matches_the_unsplit_layer(two_ranks):
    """Both ranks hold the all-reduced output; it equals the unsplit
    layer's (the shrinkage mean is summed in another order, far below the
    projection's tolerance)."""
    ref = _unsplit()
    for r in (0, 1):
        Y = two_ranks[f"row{r}"]
        err = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
        assert err < 1e-6, err
    np.testing.assert_array_equal(two_ranks["row0"], two_ranks["row1"])


def test_column_parallel_gathers_the_unsplit_layer(two_ranks):
    """Every rank computes the same scales from the whole input, so the
    gathered columns are the unsplit layer's exactly."""
    ref = _unsplit()
    for r in (0, 1):
        np.testing.assert_allclose(two_ranks[f"col{r}"], ref, rtol=0,
                                   atol=1e-12)


def test_shards_keep_groups_and_blocks_whole():
    from test_weight_quantization_b200 import tensor_parallel as tp
    assert tp.shard_channels(4096, 4, 128) == [(0, 1024), (1024, 2048),
                                               (2048, 3072), (3072, 4096)]
    # 11008 = 86 groups of 128: near-equal shards of whole groups
    sh = tp.shard_channels(11008, 8, 128)
    assert sh[0][0] == 0 and sh[-1][1] == 11008
    assert all(a % 128 == 0 and b % 128 == 0 and b > a for a, b in sh)
    assert max(b - a for a, b in sh) - min(b - a for a, b in sh) == 128
    # groups of 16 still keep 32-code blocks whole
    assert all(a % 32 == 0 for a, _ in tp.shard_channels(768, 3, 16))
    with pytest.raises(ValueError):
        tp.shard_channels(256, 3, 128)
    assert tp.shard_rows(10, 3) == [(0, 3), (3, 6), (6, 10)]
    with pytest.raises(ValueError):
        tp.shard_rows(2, 3)
