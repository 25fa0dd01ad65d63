"""Tensor-parallel sharding of the W4A16 product (bit_gemm_quant_b200.shard).

CPU: the split arithmetic, the host-side rejection of a row-parallel split
that would cut a quantization group, the group-ownership invariant (a shard
quantized on its own equals the slice of the whole matrix's quantization), and
two gloo ranks running the sharded layer end to end with the oracle standing
in for the local kernels -- their gathered / reduced Y against the unsharded
oracle product.  GPU: the library's kernels on every shard (ranks emulated one
after another on one device), combined as the collectives combine them.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from bit_gemm_quant_b200 import shard, synth
from parity import THREADS, assert_codes_equal, assert_y_elementwise

SYM, ASYM = 0, 1


# ------------------------------------------------------------ the splits --

def test_n_range_partitions_the_rows():
    for N in (1, 7, 16, 100, 4096, 11008):
        for P in (1, 2, 3, 4, 8):
            if N < P:
                with pytest.raises(shard.ShardError):
                    shard.n_range(N, P, 0)
                continue
            rs = [shard.n_range(N, P, r) for r in range(P)]
            assert rs[0][0] == 0 and rs[-1][1] == N
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_k_range_rejects_a_split_that_cuts_a_group():
    assert shard.k_range(4096, 8, 3, 128) == (1536, 2048)
    assert shard.k_range(384, 3, 2, 128) == (256, 384)
    for K, P, g in ((4096, 64, 128),     # 64 columns per device: half a group
                    (4096, 3, 128),      # K not divisible by P
                    (4096, 5, 32),
                    (1536, 4, 256),      # 384 columns: one and a half groups
                    (8192, 128, 128)):
        with pytest.raises(shard.ShardError):
            shard.k_range(K, P, 0, g)
    with pytest.raises(shard.ShardError):
        shard.k_range(4096, 2, 2, 128)   # no such rank


# -------------------------------------------------- group ownership (oracle) --

def unpack_zeros(qzeros, G):
    j = np.arange(G)
    return (qzeros[:, j // 8] >> (4 * (j % 8)).astype(np.uint32)) & np.uint32(15)


@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("mode", [SYM, ASYM])
@pytest.mark.parametrize("P", [2, 4])
@pytest.mark.parametrize("smooth", [False, True])
def test_k_shard_quantization_is_the_slice_of_the_whole(oracle_mod, g, mode, P, smooth):
    """Page 4's checklist item: with K/P a multiple of g, every group and its
    scale and zero-point belong to one device, so quantizing each device's
    columns alone reproduces the whole matrix's codes, scales and zero-points."""
    N, K = 48, 1024
    W = synth.weights(31, N, K, 0.02, 0.01, 5.0)
    s = synth.smoothing_vector(31, K) if smooth else None
    q, sc, z = oracle_mod.quant_pack(W, g, mode, s=s)
    G = K // g
    for r in range(P):
        k0, k1 = shard.k_range(K, P, r, g)
        Wl = shard.local_weight(W, "k", P, r, g)
        sl = shard.local_smoothing(s, "k", P, r, g)
        ql, scl, zl = oracle_mod.quant_pack(Wl, g, mode, s=sl)
        assert_codes_equal(ql, q[:, k0 // 8:k1 // 8], "qweight of shard %d" % r)
        assert_codes_equal(scl, sc[:, k0 // g:k1 // g], "scales of shard %d" % r)
        if mode == ASYM:
            assert_codes_equal(unpack_zeros(zl, (k1 - k0) // g), unpack_zeros(z, G)[:, k0 // g:k1 // g],
                               "zero-points of shard %d" % r)


def test_n_shard_quantization_is_the_slice_of_the_whole(oracle_mod):
    N, K, g = 50, 512, 128
    W = synth.weights(32, N, K, 0.02)
    q, sc, z = oracle_mod.quant_pack(W, g, ASYM)
    for r in range(3):
        n0, n1 = shard.n_range(N, 3, r)
        ql, scl, zl = oracle_mod.quant_pack(shard.local_weight(W, "n", 3, r, g), g, ASYM)
        assert_codes_equal(ql, q[n0:n1], "qweight")
        assert_codes_equal(scl, sc[n0:n1], "scales")
        assert_codes_equal(zl, z[n0:n1], "qzeros")


# -------------------------------------------- two gloo ranks, oracle inside --

class OracleOps:
    """The local steps on the CPU oracle (bf16 bit patterns in numpy arrays),
    results as CPU torch tensors for the gloo collectives."""

    def quant_pack(self, W, group, mode, s=None):
        return oracle.quant_pack(np.ascontiguousarray(W), group, mode, s=s)

    def gemm(self, X, packed, group, mode, N, out_f32=False):
        q, sc, z = packed
        Y = oracle.w4a16_reference(np.ascontiguousarray(X), q, sc, z, X.shape[1], group, mode)
        t = torch.from_numpy(Y)
        return t.to(torch.float32) if out_f32 else t.to(torch.bfloat16)

    def f32_to_bf16(self, Y):
        return Y.to(torch.bfloat16)

    def empty(self, shape, like, dtype):
        return torch.empty(shape, dtype=dtype)


CASE = dict(M=3, N=90, K=1024, g=128)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, split, mode, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        oracle.build()
        M, N, K, g = CASE["M"], CASE["N"], CASE["K"], CASE["g"]
        W = synth.weights(41, N, K, 0.02, 0.01, 5.0)        # every rank draws the same matrix
        X = synth.activations(42, M, K, 0.01, 40.0)
        layer = shard.ShardedW4Linear(shard.local_weight(W, split, world, rank, g), N, K, g, mode, split, world, rank,
                                      ops=OracleOps())
        Y = layer.forward(shard.local_activations(X, split, world, rank, g))
        q.put((rank, Y.float().numpy()))
    finally:
        dist.destroy_process_group()


def run_ranks(split, mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, split, mode, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=300) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def unsharded(mode):
    M, N, K, g = CASE["M"], CASE["N"], CASE["K"], CASE["g"]
    W = synth.weights(41, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(42, M, K, 0.01, 40.0)
    qw, sc, z = oracle.quant_pack(W, g, mode)
    Y = oracle.w4a16_reference(X, qw, sc, z, K, g, mode)
    Y_abs = oracle.w4a16_abs_reference(X, qw, sc, z, K, g, mode)
    return Y, Y_abs


@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_column_parallel_two_gloo_ranks(oracle_mod, mode):
    """Each rank multiplies its rows of W; the all-gather returns the whole Y on
    both ranks, equal bit for bit to the unsharded product (each output is
    the same sum, rounded once)."""
    res = run_ranks("n", mode)
    Y_ref, _ = unsharded(mode)
    want = torch.from_numpy(Y_ref).to(torch.bfloat16).float().numpy()
    for r, Y in res.items():
        assert Y.shape == want.shape
        assert np.array_equal(Y, want), "rank %d" % r


@pytest.mark.parametrize("mode", [SYM, ASYM])
def test_row_parallel_two_gloo_ranks(oracle_mod, mode):
    """Each rank multiplies its K/2 columns; the fp32 partials are all-reduced
    before the one bf16 rounding: within one bf16 rounding of the unsharded
    product plus the fp32 rounding of the two partials and their sum."""
    res = run_ranks("k", mode)
    Y_ref, Y_abs = unsharded(mode)
    for r, Y in res.items():
        assert_y_elementwise(Y.astype(np.float64), Y_ref, Y_abs, CASE["K"], "rank %d" % r)
    assert np.array_equal(res[0], res[1])


# ------------------------------------------- the library's kernels (GPU) --

@pytest.mark.gpu
@pytest.mark.parametrize("split", ["n", "k"])
@pytest.mark.parametrize("M", [1, 8, 64])
@pytest.mark.parametrize("P", [2, 4])
def test_sharded_product_on_the_library_kernels(split, M, P):
    """Every shard through w4_quant_pack and w4a16_gemm (W4_OUT_F32 for the row
    split), the P ranks emulated one after another on one GPU and combined
    the way the collectives combine them (columns side by side; fp32 partials
    added in rank order, then w4_f32_to_bf16), against the unsharded oracle."""
    from bit_gemm_quant_b200 import build
    build.build()
    import bit_gemm_quant_b200 as w4
    from parity import dev_bf16
    oracle.build()
    N, K, g, mode = 1000, 4096, 128, ASYM
    W = synth.weights(51, N, K, 0.02, 0.01, 5.0)
    X = synth.activations(52, M, K, 0.01, 40.0)
    parts = []
    for r in range(P):
        layer = shard.ShardedW4Linear(dev_bf16(shard.local_weight(W, split, P, r, g)), N, K, g, mode, split, P, r)
        if split == "k":
            # the shard's codes equal the oracle's quantization of the same columns
            ql, scl, _ = layer.packed
            oq, osc, _ = oracle.quant_pack(shard.local_weight(W, split, P, r, g), g, mode, threads=THREADS)
            assert_codes_equal(ql.cpu().numpy().view(np.uint32), oq, "qweight of shard %d" % r)
            assert_codes_equal(scl.view(torch.int16).cpu().numpy().view(np.uint16), osc, "scales of shard %d" % r)
            Xl = dev_bf16(shard.local_activations(X, split, P, r, g))
            parts.append(layer.ops.gemm(Xl, layer.packed, g, mode, N, out_f32=True))
        else:
            parts.append(layer.forward(dev_bf16(X), gather=False))
    if split == "k":
        acc = parts[0].clone()
        for p in parts[1:]:
            acc += p
        Y = w4.f32_to_bf16(acc)
    else:
        Y = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    qw, sc, z = oracle.quant_pack(W, g, mode, threads=THREADS)
    Y_ref = oracle.w4a16_reference(X, qw, sc, z, K, g, mode, threads=THREADS)
    Y_abs = oracle.w4a16_abs_reference(X, qw, sc, z, K, g, mode, threads=THREADS)
    assert_y_elementwise(Y.float().cpu().numpy().astype(np.float64), Y_ref, Y_abs, K, "split %s P=%d" % (split, P))
