"""attention_sharded: a rank's share of one batch, with the NVFP4 tensor
amax max-reduced over the process group. With a one-rank group (the GPU machine
has one GPU) the exchange is the identity, so the result is the dynamic
one-shot call's, bit for bit; the multi-rank exchange itself is checked on
the CPU with two gloo ranks (tests/test_dist_cpu.py)."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

import precision_attention_nvfp4_b200 as fp
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    yield None
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,causal", [("nvfp4", True), ("nvfp4", False), ("fp8", True)])
def test_one_rank_share_equals_the_whole_call(one_rank_group, fmt, causal):
    w = workloads.Workload("t", B=2, H=3, N=520, d=128, causal=causal, qk_format=fmt, seed=43, outliers=True)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    ref_out, ref_lse = fp.attention(q, k, v, qk_format=fmt, causal=causal)
    out, lse = fp.attention_sharded(q, k, v, qk_format=fmt, causal=causal)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))


def test_sharded_refuses_nvfp4_v(one_rank_group):
    q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fp.attention_sharded(q, q, q, pv_format="nvfp4")
