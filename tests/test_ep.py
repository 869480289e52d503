"""Expert parallelism, host side, on the CPU: the expert ranges of the ranks tile [0, E),
shard() cuts every per-expert tensor (and re-bases the CB4 outlier CSR) consistently, and
two or three gloo ranks that each sum only the pairs routed to their own experts (the
oracle standing in for the GPU) and exchange the partial sums reassemble exactly the
single-device layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp4_block_scaled_moe_b200 import MoEWeights, ep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("E,world", [(64, 2), (64, 3), (256, 4), (8, 8), (5, 2)])
def test_expert_ranges_tile_all_experts(E, world):
    got = [ep.expert_range(r, world, E) for r in range(world)]
    begin = 0
    for b, n in got:
        assert b == begin and n >= E // world and n <= E // world + 1
        begin += n
    assert begin == E
    with pytest.raises(ValueError):
        ep.expert_range(0, E + 1, E)


def _cb4_weights(E=4, H=256, I=128):
    """A CPU stand-in for a CB4 layer: every tensor's entries encode (expert, row) so the
    cut can be checked; the CSR holds e + 1 outliers in row 0 of each expert's matrix."""
    def csr(rows):
        counts = np.zeros(E * rows, np.int32)
        counts[np.arange(E) * rows] = np.arange(E) + 1
        rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        nnz = int(rp[-1])
        col = np.arange(nnz, dtype=np.int32)
        val = np.repeat(np.arange(E), np.arange(E) + 1).astype(np.int16)
        return torch.from_numpy(rp), torch.from_numpy(col), torch.from_numpy(val)
    gu_rp, gu_col, gu_val = csr(2 * I)
    dn_rp, dn_col, dn_val = csr(H)
    e_of = lambda shape: torch.arange(E, dtype=torch.int32).view(E, *([1] * (len(shape) - 1))).expand(*shape)
    rows_of = lambda rows, shape: torch.arange(E, dtype=torch.int32).repeat_interleave(rows).view(-1, 1, 1).expand(*shape)
    return MoEWeights("cb4", E, H, I, e_of((E, 2 * I, H // 2)).to(torch.uint8).contiguous(), None,
                      e_of((E, H, I // 2)).to(torch.uint8).contiguous(), None, None, None, 7.0,
                      gu_cb=rows_of(2 * I, (E * 2 * I, H // 128, 16)).to(torch.int16).contiguous(), gu_rowptr=gu_rp,
                      gu_col=gu_col, gu_val=gu_val,
                      dn_cb=rows_of(H, (E * H, I // 128, 16)).to(torch.int16).contiguous(), dn_rowptr=dn_rp,
                      dn_col=dn_col, dn_val=dn_val)


def test_shard_cuts_cb4_layer_and_rebases_csr():
    w = _cb4_weights()
    for rank, world in ((0, 2), (1, 2), (1, 3), (3, 4)):
        s = ep.shard(w, rank, world)
        b, n = ep.expert_range(rank, world, w.E)
        assert (s.expert_begin, s.local_experts, s.E) == (b, n, w.E)
        assert s.gu_codes.shape[0] == n and torch.equal(s.gu_codes[:, 0, 0].long(), torch.arange(b, b + n))
        assert s.gu_cb.shape[0] == n * 2 * w.I and int(s.gu_cb[0, 0, 0]) == b
        for pre, rows in (("gu", 2 * w.I), ("dn", w.H)):
            rp, val = getattr(s, pre + "_rowptr"), getattr(s, pre + "_val")
            assert rp.shape[0] == n * rows + 1 and int(rp[0]) == 0
            assert int(rp[-1]) == sum(e + 1 for e in range(b, b + n)) == val.shape[0]
            assert torch.equal(val.long(), torch.repeat_interleave(torch.arange(b, b + n), torch.arange(b, b + n) + 1))


def test_shard_cuts_v2a_libraries_by_expert():
    """V2a: the group records cut like scales, the per-expert libraries by expert, the CSR
    like CB4's."""
    w = _cb4_weights()
    E, I, H = w.E, w.I, w.H
    lib = lambda: torch.arange(E, dtype=torch.int16).view(E, 1, 1).expand(E, 32, 16).contiguous()   # noqa: E731
    v = MoEWeights("v2a", E, H, I, w.gu_codes, w.gu_codes.clone(), w.dn_codes, w.dn_codes.clone(), None, None, 7.0,
                   gu_cb=lib(), gu_rowptr=w.gu_rowptr, gu_col=w.gu_col, gu_val=w.gu_val,
                   dn_cb=lib(), dn_rowptr=w.dn_rowptr, dn_col=w.dn_col, dn_val=w.dn_val)
    for rank, world in ((0, 2), (1, 3), (3, 4)):
        s = ep.shard(v, rank, world)
        b, n = ep.expert_range(rank, world, E)
        assert s.gu_cb.shape == (n, 32, 16) and torch.equal(s.dn_cb[:, 0, 0].long(), torch.arange(b, b + n))
        assert torch.equal(s.gu_scales[:, 0, 0].long(), torch.arange(b, b + n))
        rp = s.gu_rowptr
        assert rp.shape[0] == n * 2 * I + 1 and int(rp[0]) == 0 and int(rp[-1]) == s.gu_val.shape[0]


def test_shard_refuses_mixed_buffers():
    w = _cb4_weights()
    m = MoEWeights("mxfp4", w.E, w.H, w.I, w.gu_codes, w.gu_codes, w.dn_codes, w.dn_codes,
                   expert_format=torch.zeros(w.E, dtype=torch.uint8))
    with pytest.raises(ValueError):
        ep.shard(m, 0, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q, fmt):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    from oracle import moe as M, routing as R
    from synth import configs as C, draws as D
    from helpers import host_small_inputs, oracle_bank
    cfg = C.small({"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5}[fmt])
    x_bits, wr, bias = host_small_inputs(cfg)
    xf = D.bf16_bits_to_f32(x_bits).astype(np.float64)
    lg = R.router_logits(xf, wr, bias)
    ids = R.topk(lg, cfg.k)
    w = R.softmax_selected(lg, ids)
    b, n = ep.expert_range(rank, world, cfg.E)
    bank = oracle_bank(cfg)
    o = np.zeros((cfg.T, cfg.k, cfg.H))
    for e in range(b, b + n):                       # only this rank's experts
        ti, jj = np.nonzero(ids == e)
        if ti.size:
            o[ti, jj] = M.expert_outputs(bank, e, xf[ti], cfg.swiglu_limit)
    part = torch.from_numpy(M.combine_slots(w, o))
    dist.barrier()
    ep.exchange(part)
    q.put((rank, part.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,world", [("mxfp4", 2), ("nvfp4", 3), ("cb4", 2)])
def test_gloo_ranks_reassemble_the_layer(fmt, world):
    import sys
    sys.path.insert(0, ROOT)
    from oracle import moe as M, routing as R
    from synth import configs as C, draws as D
    from helpers import host_small_inputs, oracle_bank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, fmt)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    cfg = C.small({"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5}[fmt])
    x_bits, wr, bias = host_small_inputs(cfg)
    xf = D.bf16_bits_to_f32(x_bits)
    y, ids, w, _ = M.moe_layer(xf, wr, bias, cfg.k, oracle_bank(cfg), cfg.swiglu_limit)
    for r in range(world):
        # the same numbers summed in another order: equal to float64 rounding
        np.testing.assert_allclose(got[r], y, rtol=1e-12, atol=1e-12 * np.abs(y).max())
