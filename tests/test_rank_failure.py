"""Failure detection across ranks, on CPU gloo ranks (no GPU, no fault).

The context-parallel forward exchanges partials with one all-gather.  When a
peer rank fails before reaching it (raises and exits) or never reaches it,
the surviving rank must not wait for good: the process group's short timeout,
or the closed connection, ends its collective with an error, which the
wrapper passes up.  The failing rank's steps are stand-ins injected through
``ops`` (the host-logic seam of the wrapper); nothing runs on a GPU.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import socket
import sys
import time

import pytest

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
TIMEOUT_S = 5


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, mode, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from scaled_dot_product_10_b200.context_parallel import PartialOps, context_parallel_attn_fwd

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=TIMEOUT_S))
    q = torch.zeros(1, 8, 2, 16)
    k = torch.zeros(1, 8, 1, 16)

    def partials(qq, kk, vv, causal, scale, diag):
        if rank == 1 and mode == "raises":
            raise RuntimeError("rank 1: injected failure before the exchange")
        if rank == 1 and mode == "stalls":
            time.sleep(6 * TIMEOUT_S)
            raise RuntimeError("rank 1: gave up after stalling")
        return torch.zeros(1, 2, 8, 16), torch.zeros(1, 2, 8)

    def merge(o_parts, lse_parts):
        return o_parts[0], lse_parts[0]

    t0 = time.monotonic()
    try:
        context_parallel_attn_fwd(q, k, k, key_offset=8 * rank, s_k_total=16,
                                  ops=PartialOps(partials, merge))
        out.put((rank, "completed", time.monotonic() - t0))
    except Exception as exc:  # noqa: BLE001 - the error itself is the result
        out.put((rank, type(exc).__name__, time.monotonic() - t0))
        if rank == 1:
            raise
    finally:
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass


@pytest.mark.parametrize("mode", ["raises", "stalls"])
def test_survivor_ends_with_an_error_when_a_peer_fails(mode):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, mode, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    deadline = time.monotonic() + 120
    while 0 not in res and time.monotonic() < deadline:
        try:
            rank, what, secs = out.get(timeout=5)
            res[rank] = (what, secs)
        except Exception:  # noqa: BLE001 - queue.Empty: keep waiting to the deadline
            pass
    procs[0].join(30)
    procs[1].join(5)
    for p in procs:  # a peer still stalled is stopped here, by its own handle
        if p.is_alive():
            p.kill()
            p.join(10)
    assert 0 in res, "the surviving rank never returned"
    what, secs = res[0]
    assert what != "completed", "the surviving rank finished without its peer's partial"
    # it learned of the failure from the collective, not from the peer's
    # eventual exit: well before a stalled peer would have arrived
    assert secs < 4 * TIMEOUT_S, f"survivor took {secs:.1f} s"
    assert procs[1].exitcode != 0
