"""Host side of the expert-parallel forward on CPU: gloo ranks exchange their counts and
each computes its plan with the library's moe_ep_plan (no GPU, no device call).

The plan must keep the one-device meaning of capacity over the whole batch: every
run's first global slot and kept rows are what the oracle's rank-major capacity
rule (`assign_slots`) gives on the concatenated batch, and what rank q sends to
rank d is exactly what rank d expects from rank q.  The two-phase plan
(moe_ep_phase_plan) splits each expert's slots at 256 * floor((n_e + 256) / 512):
per phase, what rank q sends to rank d is what d expects from q, both equal the
oracle's kept choices on each side of the split, and the phases add up to the
one-phase plan.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    # name: (S per rank, E, k, cf, seed, skew)
    "even": ((64, 64, 64, 64), 8, 2, 1.0, 1, 0.0),
    "ragged": ((17, 0, 90, 33), 16, 2, 1.25, 2, 0.0),
    "top4_skewed": ((40, 40, 40, 40), 16, 4, 0.75, 3, 2.5),
    "top8_of_32": ((25, 31, 0, 70), 32, 8, 1.0, 4, 1.0),
    "big": ((700, 900, 800, 600), 8, 2, 1.25, 5, 0.5),        # n_e up to C = 938: both phases non-empty
}


def _ids(S_all, E, k, seed, skew):
    """Per-rank expert ids from seeded logits routed by the oracle (ties: lower index)."""
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((sum(S_all), E)).astype(np.float32)
    logits += skew * np.log(1.0 / (np.arange(E) + 1.0)).astype(np.float32)
    ids = O.top_k(logits, k)
    cuts = np.cumsum((0,) + tuple(S_all))
    return ids, [ids[cuts[q]:cuts[q + 1]] for q in range(len(S_all))]


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gshard_top_gating_b200 import _lib as L
        S_all, E, k, cf, seed, skew = CASES[case]
        S_all = S_all[:world] if world < len(S_all) else S_all
        _, mine = _ids(S_all, E, k, seed, skew)
        ids = mine[rank]
        # this rank's counts: rank-r demand of each expert
        cnt = np.zeros((k, E), dtype=np.int64)
        for r in range(k):
            cnt[r] = np.bincount(ids[:, r], minlength=E)
        gathered = [torch.zeros(k * E + 1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(np.concatenate([cnt.ravel(), [len(ids)]])))
        counts = np.stack([g_[:-1].numpy().reshape(k, E) for g_ in gathered])
        S = np.array([int(g_[-1]) for g_ in gathered])
        C, send, recv, base, kept = L.moe_ep_plan(world, rank, E, k, cf, counts, S)
        # what rank d receives from this rank must be what this rank sends to d
        got = torch.zeros(world, dtype=torch.int64)
        dist.all_to_all_single(got, torch.from_numpy(send.copy()))
        send2, recv2, split = L.moe_ep_phase_plan(world, rank, E, k, cf, counts, S, 2)
        got2 = []
        for ph in range(2):                    # the same check for each phase's exchange
            g2 = torch.zeros(world, dtype=torch.int64)
            dist.all_to_all_single(g2, torch.from_numpy(send2[ph].copy()))
            got2.append(g2.numpy())
        q.put((rank, C, send, recv, base, kept, got.numpy(), counts, S, send2, recv2, split, np.stack(got2)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, "even"), (4, "even"), (4, "ragged"), (4, "top4_skewed"),
                                        (4, "top8_of_32"), (2, "top8_of_32"), (4, "big"), (2, "big")])
def test_exchange_plan_matches_the_one_device_capacity_rule(world, case):
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([qu.get(timeout=240) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0

    S_all, E, k, cf, seed, skew = CASES[case]
    S_all = S_all[:world]
    ids, _ = _ids(S_all, E, k, seed, skew)
    S_tot = sum(S_all)
    C = O.capacity(S_tot, E, k, cf)
    slot, cnt_tot = O.assign_slots(ids, E, C)
    pos, _ = O.assign_slots(ids, E, S_tot * k + 1)        # positions with nothing dropped
    El = E // world
    owner = np.repeat(np.arange(len(S_all)), S_all)
    n_e = np.minimum(cnt_tot, C)
    split_ref = 256 * ((n_e + 256) // 512)
    assert np.all(split_ref <= n_e)
    for rank, C_got, send, recv, base, kept, got, counts, S, send2, recv2, split, got2 in res:
        assert np.array_equal(split, split_ref)
        # per phase: the exchange is consistent, matches the oracle's kept choices on
        # each side of the split, and the two phases add up to the one-phase plan
        assert np.array_equal(got2, recv2)
        assert np.array_equal(send2.sum(axis=0), send) and np.array_equal(recv2.sum(axis=0), recv)
        ph_of = np.where(slot >= 0, (slot >= split_ref[np.clip(ids, 0, E - 1)]).astype(int), -1)
        for ph in range(2):
            for d in range(world):
                e_d = (ids // El == d)
                assert send2[ph, d] == int(np.sum((ph_of == ph) & e_d & (owner == rank)[:, None]))
                assert recv2[ph, d] == int(np.sum((ph_of == ph) & (ids // El == rank) & (owner == d)[:, None]))
        assert C_got == C
        assert np.array_equal(S, S_all)
        # what every rank d sends here (exchanged by gloo) is what this rank expects from d
        assert np.array_equal(got, recv)
        assert np.array_equal(recv, [res[d][2][rank] for d in range(world)])
        for q_ in range(world):
            for r in range(k):
                for e in range(E):
                    sel = np.nonzero((owner == q_) & (ids[:, r] == e))[0]
                    assert counts[q_, r, e] == len(sel)
                    if len(sel):                          # the run starts at its first choice's position
                        assert base[q_, r, e] == pos[sel[0], r]
                        assert np.array_equal(pos[sel, r], base[q_, r, e] + np.arange(len(sel)))
                    assert kept[q_, r, e] == int(np.sum(slot[sel, r] >= 0))
        # rows this rank sends to d: its kept choices of d's experts; receives: all ranks' of its own
        for d in range(world):
            e_d = (ids // El == d)
            assert send[d] == int(np.sum((slot >= 0) & e_d & (owner == rank)[:, None]))
        mine = ids // El == rank
        assert recv.sum() == int(np.sum((slot >= 0) & mine))
    # every expert keeps min(demand, C) rows in total
    kept0 = res[0][5]
    assert np.array_equal(kept0.sum(axis=(0, 1)), np.minimum(cnt_tot, C))


def test_plan_rejects_inconsistent_counts():
    from gshard_top_gating_b200 import _lib as L
    counts = np.array([[[2, 1]], [[0, 3]]], dtype=np.int64)      # G=2, k=1, E=2
    C, send, recv, base, kept = L.moe_ep_plan(2, 0, 2, 1, 1.0, counts, [3, 3])
    assert C == 3 and list(send) == [2, 1] and list(recv) == [2, 0]
    assert base[:, 0, 1].tolist() == [0, 1] and kept[:, 0, 1].tolist() == [1, 2]
    with pytest.raises(L.MoeError) as ei:                       # rank 1's counts do not sum to S
        L.moe_ep_plan(2, 0, 2, 1, 1.0, counts, [3, 4])
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoeError):
        L.moe_ep_plan(2, 0, 3, 1, 1.0, np.zeros((2, 1, 3)), [0, 0])   # E not a multiple of G
    with pytest.raises(L.MoeError):
        L.moe_ep_plan(2, 2, 2, 1, 1.0, counts, [3, 3])             # g out of range
    with pytest.raises(L.MoeError) as ei:
        L.moe_ep_phase_plan(2, 0, 2, 1, 1.0, counts, [3, 3], 3)   # one or two phases only
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    send1, recv1, split1 = L.moe_ep_phase_plan(2, 0, 2, 1, 1.0, counts, [3, 3], 1)
    assert send1.tolist() == [[2, 1]] and recv1.tolist() == [[2, 0]] and split1.tolist() == [2, 3]
