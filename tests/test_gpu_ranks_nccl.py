"""The multi-GPU call's torch.distributed path on a one-process NCCL group.

With one GPU per run here, the group has a single rank (P = 1): NCCL's
all_to_all_single and all_gather_into_tensor then copy each send view into
the receive view, which checks that the collectives accept the exchange
plan's CUDA views (uint8 codes, int32 parameters, uneven split lists) and
order with the kernels on torch's current stream; and EchoRank.allreduce
gives the oracle's P = 1 result. The exchange logic between several ranks
is covered on gloo CPU ranks (test_multirank_exchange.py) and the rank
kernels with P > 1 against the oracle (test_gpu_ranks.py).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle as O
import bit_error_compensated_group_b200 as E
from parity import padded, random_inputs, u16

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


def test_collectives_accept_the_plan(nccl_group):
    n, group = 10000, 128
    rk = E.EchoRank(n, 1, 0, group, 8, True)
    try:
        for bits in (4, 8):
            plan = rk.plan(bits)
            plan.send_codes.copy_(torch.randint(0, 256, plan.send_codes.shape, dtype=torch.uint8, device="cuda"))
            plan.send_params.copy_(torch.randint(-2**31, 2**31 - 1, plan.send_params.shape, dtype=torch.int32,
                                                 device="cuda"))
            plan.gsend_codes.copy_(torch.randint(0, 256, plan.gsend_codes.shape, dtype=torch.uint8, device="cuda"))
            plan.gsend_params.copy_(torch.randint(-2**31, 2**31 - 1, plan.gsend_params.shape, dtype=torch.int32,
                                                  device="cuda"))
            E.exchange_all_to_all(plan)
            E.exchange_all_gather(plan)
            torch.cuda.synchronize()
            assert torch.equal(plan.recv_codes, plan.send_codes)
            assert torch.equal(plan.recv_params, plan.send_params)
            assert torch.equal(plan.grecv_codes, plan.gsend_codes)
            assert torch.equal(plan.grecv_params, plan.gsend_params)
    finally:
        rk.close()


def test_allreduce_one_rank_matches_the_oracle(nccl_group):
    n, group = 70001, 64
    G = -(-n // group)
    rk = E.EchoRank(n, 1, 0, group, 4, True)
    try:
        x = random_inputs(1, n, 99, 3.0)
        xd = x[0].cuda()
        out = torch.empty_like(xd)
        el = np.zeros((1, G * group), np.float32)
        es = np.zeros((1, G * group), np.float32)
        xb = padded(u16(x), G * group)
        for call in range(2):
            rk.allreduce(xd, out, 4, 1.0, 0.05, 0.5, 0.5)
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=4, e_long=el, e_short=es)
            assert np.array_equal(u16(out), orc.y[0, :n]), f"call {call}"
            L, S = rk.ema_views()
            assert np.array_equal(L.cpu().numpy(), el[0, :n]) and np.array_equal(S.cpu().numpy(), es[0, :n])
    finally:
        rk.close()
