"""Failure detection of the multi-rank path on CPU ranks (gloo): one rank fails
before the first exchange (an exception in its prologue), and the other rank's
pending all-to-all ends with an error within the process group's short timeout
instead of waiting for ever.  The failure is made on the host; nothing runs on
a GPU."""
import os
import socket
import time
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from video_diffusion_transformer_h3attn_b200 import ulysses

PG_TIMEOUT_S = 5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _copy_prologue(q_in, k_in, q_out, k_out, *args):
    q_out.copy_(q_in)
    k_out.copy_(k_in)


def _failing_prologue(*args):
    raise RuntimeError("injected failure before the exchange")


def _never_called(*args):
    raise AssertionError("attention must not run after a failed exchange")


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=PG_TIMEOUT_S))
    t0 = time.monotonic()
    try:
        n, H, d = 10, 4, 8
        sizes = ulysses.shard_sizes(n, world)
        x = torch.zeros((sizes[rank], H, d), dtype=torch.bfloat16)
        ulysses.ulysses_attention(x, x.clone(), x.clone(), sizes,
                                  prologue_fn=_failing_prologue if rank == 1 else _copy_prologue,
                                  attention_fn=_never_called)
        out[rank] = ("ok", time.monotonic() - t0)
    except Exception as exc:  # the failure under test
        out[rank] = ("error: %s" % type(exc).__name__, time.monotonic() - t0)
    finally:
        dist.destroy_process_group()


def test_a_failed_rank_ends_the_others_exchange_with_an_error():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()  # this test's own child, by its handle
        p.join()
    assert not alive, "a rank hung after its peer failed"
    assert out[1][0].startswith("error"), "the failing rank must report its error: %r" % (out[1],)
    assert out[0][0].startswith("error"), "the surviving rank's exchange must fail, not finish: %r" % (out[0],)
    assert out[0][1] < 60.0, "the surviving rank waited %.1f s" % out[0][1]
