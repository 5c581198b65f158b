"""The expert cache's bookkeeping (host only, no GPU): sizes, the reuse order
of its slots, and moe_cache_admit against an independent model of the policy
the header states (free slots first, lowest index on ties; otherwise the least
recently used slot; slots named by the current call are never reused in it)."""
import ctypes as C

import numpy as np
import pytest

import quantized_expert_decode_moe_b200 as qm
from test_abi_host import fake_layer


def make_cache(E=16, slots=3, H=256, I=128, bits=4):
    lay = fake_layer(hidden=H, inter=I, n_experts=E, bits=bits)
    L = qm.lib()
    d, h = C.c_size_t(0), C.c_size_t(0)
    assert L.moe_cache_size(C.byref(lay), slots, C.byref(d), C.byref(h)) == 0
    host = (qm._Expert * E)(*[qm._Expert(*[qm._QMat(0x1000, 0x1000, 0x1000) for _ in range(3)]) for _ in range(E)])
    state = np.zeros((h.value + 7) // 8, dtype=np.uint64)
    dev = C.c_void_p(0x10000000)   # never touched by init or admit
    assert L.moe_cache_init(C.byref(lay), C.cast(host, C.c_void_p), slots, dev, d.value,
                            C.c_void_p(state.ctypes.data), state.nbytes) == 0
    return lay, host, state, d.value


def admit(state, ids):
    ids = np.asarray(ids, dtype=np.int32)
    slot, missed = np.empty_like(ids), np.empty_like(ids)
    rc = qm.lib().moe_cache_admit(C.c_void_p(state.ctypes.data), C.c_void_p(ids.ctypes.data), ids.size,
                                  C.c_void_p(slot.ctypes.data), C.c_void_p(missed.ctypes.data))
    return rc, slot.tolist(), missed.tolist()


def stats(state):
    h, m, b = C.c_uint64(), C.c_uint64(), C.c_uint64()
    assert qm.lib().moe_cache_stats(C.c_void_p(state.ctypes.data), C.byref(h), C.byref(m), C.byref(b)) == 0
    return h.value, m.value


def test_sizes():
    """Device bytes = the expert table (E descriptors, 256-byte aligned) + slots x the nine arrays of
    an expert, each 256-byte aligned."""
    H, I, E, slots = 256, 128, 16, 3
    lay = fake_layer(hidden=H, inter=I, n_experts=E, bits=4)
    d, h = C.c_size_t(0), C.c_size_t(0)
    assert qm.lib().moe_cache_size(C.byref(lay), slots, C.byref(d), C.byref(h)) == 0
    a = lambda v: (v + 255) // 256 * 256
    q, sc = I * H // 2, I * (H // 64) * 2   # the same for gate, up and down (square in codes)
    per = 3 * (a(q) + 2 * a(sc))
    assert d.value == a(E * C.sizeof(qm._Expert)) + slots * per
    assert h.value > 0
    assert qm.lib().moe_cache_size(C.byref(lay), 0, C.byref(d), C.byref(h)) == 1


def test_reuse_order():
    _, _, st, _ = make_cache(E=16, slots=3)
    assert admit(st, [5, 7, 5]) == (0, [0, 1, 0], [1, 1, 0])
    assert stats(st) == (0, 2)
    assert admit(st, [7, 9]) == (0, [1, 2], [0, 1])         # 7 resident; 9 takes the free slot
    assert stats(st) == (1, 3)
    assert admit(st, [3]) == (0, [0], [1])                  # full: slot 0 (expert 5) is the oldest
    assert admit(st, [5, 9]) == (0, [1, 2], [1, 0])         # 9 resident (slot 2); 5 takes slot 1 (expert 7, older than 3)
    assert stats(st) == (2, 5)
    assert admit(st, [1, 2, 3, 4])[0] == 2                  # four distinct experts, three slots
    assert admit(st, [16])[0] == 1                           # id out of range
    assert admit(st, [-1])[0] == 1


def test_uninitialised_state_rejected():
    st = np.zeros(4096, dtype=np.uint64)
    assert admit(st, [1])[0] == 1


def lru_model(E, slots, calls):
    """The policy as the header states it, written directly: per call, resident ids are hits;
    each missing expert (first occurrence) takes a free slot (lowest index) or else the least
    recently used slot not named by this call (lowest index on ties)."""
    owner = [-1] * slots
    last = [0] * slots
    out = []
    for c, ids in enumerate(calls, start=1):
        where = {owner[s]: s for s in range(slots) if owner[s] >= 0}
        used = {where[e] for e in ids if e in where}
        for s in used:
            last[s] = c
        slot, missed = [], []
        for e in ids:
            if e in where:
                slot.append(where[e])
                missed.append(0)
                continue
            free = [s for s in range(slots) if owner[s] < 0]
            if free:
                s = free[0]
            else:
                cand = [s for s in range(slots) if s not in used]
                s = min(cand, key=lambda q: (last[q], q))
            if owner[s] >= 0:
                del where[owner[s]]
            owner[s] = e
            where[e] = s
            last[s] = c
            used.add(s)
            slot.append(s)
            missed.append(1)
        out.append((slot, missed))
    return out


@pytest.mark.parametrize("E,slots,k", [(16, 3, 2), (64, 8, 3), (512, 24, 3)])
def test_admit_matches_the_policy(E, slots, k):
    rng = np.random.default_rng(E + slots)
    calls = []
    for _ in range(300):
        T = int(rng.integers(1, max(2, slots // k) + 1))
        ids = rng.integers(0, E if rng.random() < 0.5 else min(E, 2 * slots), size=T * k).tolist()
        if len(set(ids)) <= slots:
            calls.append(ids)
    _, _, st, _ = make_cache(E=E, slots=slots)
    model = lru_model(E, slots, calls)
    hits = misses = 0
    for ids, (slot, missed) in zip(calls, model):
        rc, s, m = admit(st, ids)
        assert rc == 0 and s == slot and m == missed, ids
        distinct = len(set(ids))
        misses += sum(missed)
        hits += distinct - sum(missed)
    assert stats(st) == (hits, misses)
