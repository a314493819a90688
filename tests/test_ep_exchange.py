"""Expert-parallel exchange on CPU: three gloo ranks run the package's
all-to-all dispatch and combine helpers (binding.ep_exchange / ep_return) on
row spaces laid out the way moe_ep_dispatch lays them out ("Appendix C -
Acronyms & Symbols", "Capacity & communication": each device holds E/G experts;
tokens reach them by an all-to-all dispatch and return by an all-to-all
combine). Every rank must receive exactly the segments of its own experts,
source-major, and every source must get back each row's result at the row it
sent. The expert MLPs themselves run on the GPU (test_parity_gpu.py emulates
the ranks on one device)."""
from __future__ import annotations

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

G, E, D, O = 3, 6, 5, 4
El = E // G


def _expert_rows(rank: int):
    rng = np.random.default_rng(100 + rank)
    rows = (rng.integers(0, 4, size=E) * 32).tolist()  # padded segments, some empty
    rows[rank] = 0  # one empty expert segment per rank
    return rows


def _send_rows(rank: int, rows):
    # Row j of expert e's segment carries (source, expert, j) in its first columns.
    out = []
    for e in range(E):
        for j in range(rows[e]):
            r = np.zeros(D, np.float32)
            r[:3] = (rank, e, j)
            out.append(r)
    return torch.tensor(np.array(out, np.float32).reshape(-1, D))


def _expert_fn(x: torch.Tensor) -> torch.Tensor:
    # A stand-in for an expert: a fixed function of the received row.
    return torch.stack([x[:, 0] * 10 + x[:, 1], x[:, 2] + 0.5, x[:, 1], x[:, 0]], dim=1)


def _rank_main(rank: int, port: int, result_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=G)
    try:
        from sparse_mixture_experts_gate_b200.binding import ep_exchange, ep_return, ep_send_splits
        rows = _expert_rows(rank)
        send = _send_rows(rank, rows)
        recv, counts, send_splits, recv_splits = ep_exchange(send, rows, G)
        # Received: for each source s, the segments of experts rank*El .. in order.
        want = []
        for s_ in range(G):
            rs = _expert_rows(s_)
            assert counts[s_].tolist() == rs[rank * El:(rank + 1) * El]
            for e in range(rank * El, (rank + 1) * El):
                for j in range(rs[e]):
                    want.append([s_, e, j])
        got = recv[:, :3].numpy().astype(int).tolist()
        assert got == want, f"rank {rank}: received rows out of order"
        assert send_splits == ep_send_splits(rows, G) and sum(recv_splits) == recv.shape[0]
        # Expert compute on the received rows, then back to the sources.
        back = torch.full((send.shape[0], O), -1.0)
        ep_return(_expert_fn(recv), back, send_splits, recv_splits)
        assert torch.equal(back, _expert_fn(send)), f"rank {rank}: results not back at their rows"
        open(os.path.join(result_dir, f"ok{rank}"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_exchange_three_gloo_ranks(tmp_path):
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=G, join=True)
    assert all((tmp_path / f"ok{r}").exists() for r in range(G))
