"""The data-parallel plumbing (gradient all-reduce, max-over-ranks timing,
token shards that share the weights) with two gloo ranks on CPU."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from nvfp4_bit_precision_quantize_b200 import dp
    from nvfp4_bit_precision_quantize_b200 import workloads as W
    dp.init("gloo", timeout_s=60)
    g1 = torch.full((4, 3), float(rank + 1))
    g2 = torch.arange(6, dtype=torch.float32) * (rank + 1)
    dp.allreduce_grads([g1, g2])
    slowest = dp.max_over_ranks(1.5 + rank)
    w = W.mlp(seed=5, M=64, H=32, F=48, data_seed=dp.shard_data_seed(5, rank))
    dp.barrier()
    q.put((rank, g1.tolist(), g2.tolist(), slowest, {k: v.tolist() for k, v in w.items()}))
    dp.finish()


def test_two_rank_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, g1, g2, slowest, _ in res:
        assert g1 == [[3.0] * 3] * 4
        assert g2 == [float(3 * i) for i in range(6)]
        assert slowest == 2.5
    w0, w1 = res[0][4], res[1][4]
    assert w0["W1"] == w1["W1"] and w0["W2"] == w1["W2"]      # one model on every rank
    assert w0["X"] != w1["X"] and w0["dY2"] != w1["dY2"]      # each rank its own tokens


def _mlp_inputs(rank, M=64, H=64, F=128):
    from nvfp4_bit_precision_quantize_b200 import dp
    from nvfp4_bit_precision_quantize_b200 import workloads as W
    w = W.mlp(seed=5, M=M, H=H, F=F, data_seed=dp.shard_data_seed(5, rank))
    return {k: W.bits_to_torch_bf16(v) for k, v in w.items()}


def _mlp_worker(rank, world, port, q):
    """One rank of a reduced MLP step: the step's own call sequence (mlp.MlpStep) with
    the oracle as the compute (tests/cpu_stand_in.py) and the overlapped gradient
    exchange of dp.GradExchange."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import cpu_stand_in
    from nvfp4_bit_precision_quantize_b200 import dp
    from nvfp4_bit_precision_quantize_b200.mlp import MlpStep
    dp.init("gloo", timeout_s=60)
    step = MlpStep(_mlp_inputs(rank), lib=cpu_stand_in)
    ex = dp.GradExchange()

    def ready(name, t):
        cpu_stand_in.calls.append("exchange " + name)
        ex.ready(name, t)

    step.step(grad_ready=ready)
    ex.wait()
    dp.barrier()
    q.put((rank, list(cpu_stand_in.calls), ex.order, step.dW1.clone(), step.dW2.clone()))
    dp.finish()


def test_two_rank_mlp_step_exchange():
    """Each rank runs the MLP step on its own token shard; dW2's all-reduce is issued
    as soon as its GEMM is queued (before the up-projection's backward starts), dW1's
    after the last GEMM, and both end up as the sum of the ranks' local gradients."""
    import cpu_stand_in
    from nvfp4_bit_precision_quantize_b200.mlp import MlpStep
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_mlp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    local = []
    for rank in range(2):  # each shard's gradients without an exchange
        st = MlpStep(_mlp_inputs(rank), lib=cpu_stand_in)
        st.step()
        local.append((st.dW1, st.dW2))
    for rank, calls, order, dW1, dW2 in res:
        assert order == ["dW2", "dW1"]
        gemms = [i for i, c in enumerate(calls) if c.startswith("gemm")]
        assert len(gemms) == 6
        i2 = calls.index("exchange dW2")
        assert calls[i2 - 1] == "gemm"
        assert sum(1 for i in gemms if i > i2) == 2                          # overlaps the up-projection bwd
        assert calls[-1] == "exchange dW1" and calls[-2] == "gemm"
        assert torch.equal(dW1, local[0][0] + local[1][0])
        assert torch.equal(dW2, local[0][1] + local[1][1])
        assert not torch.equal(local[0][0], local[1][0])                    # the shards differ


def test_rank0_keeps_the_single_gpu_workload():
    from nvfp4_bit_precision_quantize_b200 import dp
    from nvfp4_bit_precision_quantize_b200 import workloads as W
    a = W.mlp(seed=5, M=64, H=32, F=48)
    b = W.mlp(seed=5, M=64, H=32, F=48, data_seed=dp.shard_data_seed(5, 0))
    for k in a:
        assert (a[k] == b[k]).all(), k
