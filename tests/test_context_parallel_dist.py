"""Context-parallel orchestration on CPU: gloo ranks (2 and 3) each hold one segment of
the sequence and run ssd_fwd_context_parallel with per-rank steps computed in fp64 on the
host (the local forward is the oracle's recurrence; decay sums, the exclusive scan over
ranks and the state-to-output correction restate the decomposition of the sequence-
parallel scheme). The gathered outputs and the last rank's end state must equal the
oracle run over the whole, unsplit sequence: this pins the partition, the collective,
which rank takes h0 and which ranks correct."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BLK = 128


class HostSteps:
    """fp64 host versions of the four per-rank steps (torch CPU tensors in and out)."""

    def fwd(self, x, dt, A, B, C, D, h0, chunk):
        import oracle

        y, hf = oracle.recurrent(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                                 None if D is None else D.numpy(), None if h0 is None else h0.numpy())
        return torch.from_numpy(np.ascontiguousarray(y)), torch.from_numpy(np.ascontiguousarray(hf))

    def decay(self, dt, A):
        a = dt.numpy() * A.numpy()[None, None, :]                    # [B, L, H]
        Bsz, L, H = a.shape
        nblk = max((L + BLK - 1) // BLK, 1)
        bd = np.zeros((Bsz, H, nblk))
        for k in range(nblk):
            bd[:, :, k] = a[:, k * BLK:(k + 1) * BLK, :].sum(axis=1)
        return torch.from_numpy(bd), torch.from_numpy(a.sum(axis=1))

    def combine(self, states, totals, rank):
        S = torch.zeros_like(states[0])
        for q in range(rank):
            S = torch.exp(totals[q])[:, :, None, None] * S + states[q]
        return S, torch.exp(totals[rank])[:, :, None, None] * S + states[rank]

    def correct(self, dt, A, C, block_decay, s_in, y):
        a = dt.numpy() * A.numpy()[None, None, :]
        cum = np.cumsum(a, axis=1)                                   # through token t, inclusive
        H, G = a.shape[2], C.shape[2]
        Cg = C.numpy()[:, :, np.arange(H) // (H // G), :]            # [B, L, H, N]
        y += torch.from_numpy(np.exp(cum)[..., None] * np.einsum("blhn,bhpn->blhp", Cg, s_in.numpy()))
        return y


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, L, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from state_space_sequence_chunked_b200 import inputs
    from state_space_sequence_chunked_b200.context_parallel import segment_bounds, ssd_fwd_context_parallel

    dist.init_process_group("gloo", rank=rank, world_size=ws)
    d = inputs.draw(inputs.WORKLOADS["tiny_fp32"], batch=2, seqlen=L, seed=11, h0_std=0.5)
    lo, hi = segment_bounds(L, ws, rank)
    seg = lambda k: torch.from_numpy(np.ascontiguousarray(d[k].value[:, lo:hi]))
    full = lambda k: torch.from_numpy(d[k].value)
    y, h_end = ssd_fwd_context_parallel(seg("x"), seg("dt"), full("A"), seg("B"), seg("C"), full("D"),
                                        full("h0") if rank == 0 else None, chunk=64, steps=HostSteps())
    q.put((rank, lo, hi, y.numpy(), h_end.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("ws,L", [(2, 300), (3, 257)])
def test_gloo_ranks_reproduce_the_unsplit_sequence(ws, L):
    sys.path.insert(0, ROOT)
    import oracle
    from state_space_sequence_chunked_b200 import inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, L, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = []
    import time
    deadline = time.time() + 300
    while len(res) < ws:
        assert time.time() < deadline, "ranks did not report"
        try:
            res.append(q.get(timeout=2))
        except Exception:
            assert all(p.exitcode in (None, 0) for p in procs), [p.exitcode for p in procs]
    res.sort(key=lambda r: r[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    d = inputs.draw(inputs.WORKLOADS["tiny_fp32"], batch=2, seqlen=L, seed=11, h0_std=0.5)
    yr, hr = oracle.recurrent(d["x"].value, d["dt"].value, d["A"].value, d["B"].value, d["C"].value,
                              d["D"].value, d["h0"].value)
    assert [r[1] for r in res] == [0] + [r[2] for r in res[:-1]] and res[-1][2] == L   # contiguous, in order
    y = np.concatenate([r[3] for r in res], axis=1)
    scale = np.max(np.abs(yr))
    assert np.max(np.abs(y - yr)) <= 1e-10 * scale
    assert np.max(np.abs(res[-1][4] - hr)) <= 1e-10 * np.max(np.abs(hr))
    # each rank's end state is the true state at its segment's end
    for r in res[:-1]:
        sl = lambda k: np.ascontiguousarray(d[k].value[:, :r[2]])
        _, hmid = oracle.recurrent(sl("x"), sl("dt"), d["A"].value, sl("B"), sl("C"), d["D"].value, d["h0"].value)
        assert np.max(np.abs(r[4] - hmid)) <= 1e-10 * np.max(np.abs(hmid))


def test_segment_bounds_cover_the_sequence():
    sys.path.insert(0, ROOT)
    from state_space_sequence_chunked_b200.context_parallel import segment_bounds

    for L in (0, 1, 7, 128, 1000):
        for ws in (1, 2, 3, 8):
            b = [segment_bounds(L, ws, r) for r in range(ws)]
            assert b[0][0] == 0 and b[-1][1] == L
            assert all(b[i][1] == b[i + 1][0] for i in range(ws - 1))
            assert max(h - l for l, h in b) - min(h - l for l, h in b) <= 1
