"""A sequence split across ranks (selective_state_space_22_b200.seqpar).

CPU (gloo, world size 2): the orchestration -- which rank starts from the
initial state, the all-gather of (end state, total log-decay), the fold of the
ranks before each one -- with the three steps done by the fp64 oracle, against
the oracle's scan of the whole sequence.

GPU (one process): the library's steps on slices of one sequence as R ranks
would run them (state-only scan of every slice, fold, full scan from the folded
state), against the oracle's scan of the whole sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, oracle_scan, rel_err


class OracleOps:
    """The three steps of the split, by the fp64 oracle (CPU tensors in and out)."""

    def final_state(self, x, dt, A, B, init_state, chunk_size):
        n = lambda t: None if t is None else np.ascontiguousarray(t.double().numpy())
        _, fs = oracle.scan(n(x), n(dt), n(A), n(B), n(B), None, n(init_state))
        lam = n(A)[None, :] * n(dt).sum(axis=1)
        return torch.from_numpy(fs), torch.from_numpy(lam)

    def fold(self, states, log_decay):
        h = states[0].clone()
        for j in range(1, states.shape[0]):
            h = torch.exp(log_decay[j])[:, :, None, None] * h + states[j]
        return h

    def scan(self, x, dt, A, B, C, D, init_state, chunk_size):
        n = lambda t: None if t is None else np.ascontiguousarray(t.double().numpy())
        y, fs = oracle.scan(n(x), n(dt), n(A), n(B), n(C), n(D), n(init_state))
        return torch.from_numpy(y), torch.from_numpy(fs)


SHAPE = inputs.ScanShape("seqpar", 2, 301, 3, 8, 1, 4, 64, "f32", init_state=True, seed=55)


def _slices(T, world):
    cuts = [T * r // world for r in range(world + 1)]
    return list(zip(cuts[:-1], cuts[1:]))


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    from selective_state_space_22_b200.seqpar import scan_fwd_sequence_parallel

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    inp = inputs.scan_inputs(SHAPE)
    t0, t1 = _slices(SHAPE.seqlen, world)[rank]
    sl = lambda t: t[:, t0:t1].contiguous()
    y, fs = scan_fwd_sequence_parallel(sl(inp["x"]), sl(inp["dt"]), inp["A"], sl(inp["B"]), sl(inp["C"]),
                                       inp["D"], inp["init_state"] if rank == 0 else None, chunk_size=64,
                                       ops=OracleOps())
    np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
    np.save(os.path.join(out_dir, f"f{rank}.npy"), fs.numpy())
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_and_fold_on_cpu_ranks(tmp_path, world):
    import torch.multiprocessing as mp

    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    y = np.concatenate([np.load(tmp_path / f"y{r}.npy") for r in range(world)], axis=1)
    y_ref, fs_ref = oracle_scan(inputs.scan_inputs(SHAPE))
    assert y.shape == y_ref.shape
    assert rel_err(y, y_ref) < 1e-12
    assert rel_err(np.load(tmp_path / f"f{world - 1}.npy"), fs_ref) < 1e-12
    # every rank's end state is the true state at the end of its slice
    for r, (_, t1) in enumerate(_slices(SHAPE.seqlen, world)[:-1]):
        w = inputs.widen_all(inputs.scan_inputs(SHAPE))
        c = lambda a: np.ascontiguousarray(a[:, :t1])
        _, f_true = oracle.scan(c(w["x"]), c(w["dt"]), w["A"], c(w["B"]), c(w["C"]), w["D"], w["init_state"])
        assert rel_err(np.load(tmp_path / f"f{r}.npy"), f_true) < 1e-12


@pytest.mark.gpu
@pytest.mark.parametrize("io,T,R", [("bf16", 4 * 640 + 77, 4), ("f32", 1000, 3), ("bf16", 2 * 128, 2)])
def test_slices_on_one_device(io, T, R):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import selective_state_space_22_b200 as ssd

    shape = inputs.ScanShape("seqpar-gpu", 2, T, 8, 64, 1, 128, 128, io, init_state=True, seed=T)
    inp = inputs.scan_inputs(shape)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    cuts = _slices(T, R)
    sl = lambda t, r: t[:, cuts[r][0]:cuts[r][1]].contiguous()
    S, lam = [], []
    for r in range(R):
        s_r, l_r = ssd.ssd_scan_final_state(sl(d["x"], r), sl(d["dt"], r), d["A"], sl(d["B"], r),
                                            d["init_state"] if r == 0 else None, chunk_size=128)
        S.append(s_r)
        lam.append(l_r)
    ys, fin = [], None
    for r in range(R):
        h_in = d["init_state"] if r == 0 else ssd.ssd_fold_states(torch.stack(S[:r]), torch.stack(lam[:r]))
        y_r, fin = ssd.ssd_scan_fwd(sl(d["x"], r), sl(d["dt"], r), d["A"], sl(d["B"], r), sl(d["C"], r), d["D"],
                                    h_in, chunk_size=128)
        ys.append(y_r)
    ssd.ssd_get_device_status()
    y = torch.cat(ys, 1).float().cpu().numpy()
    y_ref, fs_ref = oracle_scan(inp)
    tol = TOL_BF16 if io == "bf16" else TOL_F32
    assert rel_err(y, y_ref) <= tol
    assert rel_err(fin.cpu().numpy(), fs_ref) <= tol
    # the slice log-decay is A * sum(dt) over the slice
    lam0 = inp["A"].double()[None, :] * inp["dt"][:, cuts[0][0]:cuts[0][1]].double().sum(1)
    assert rel_err(lam[0].cpu().numpy(), lam0.numpy()) < 1e-6


@pytest.mark.gpu
@pytest.mark.parametrize("b,T,H", [(1, 2048, 4), (2, 700, 8), (1, 128 * 37 + 5, 2)])
def test_state_only_form_matches_the_full_scan_bitwise(b, T, H):
    """The state-only form (its own kernel instance, W built by another warpgroup
    into another buffer) forms the same bf16 W tiles and chunk-state products as
    the full scan, in the same order: the final states agree bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import selective_state_space_22_b200 as ssd

    shape = inputs.ScanShape("state-only-vs-full", b, T, H, 64, 1, 128, 128, "bf16", init_state=True, seed=T + H)
    inp = inputs.scan_inputs(shape)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    _, f_full = ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], chunk_size=128)
    f_only, _ = ssd.ssd_scan_final_state(d["x"], d["dt"], d["A"], d["B"], d["init_state"], chunk_size=128)
    ssd.ssd_get_device_status()
    assert torch.equal(f_only, f_full)
