"""The exchange-volume accounting (host only, CPU): closed forms, and the
payload ratio the SGLang "Sequence Parallelism" page states for kv_gather
against Ulysses: P/2 per rank -- about equal at SP2, about 2x at SP4, 4x at
SP8."""
import pytest

from context_attention_long_b200 import api, build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


@pytest.mark.parametrize("P", [2, 4, 8])
def test_kv_gather_over_ulysses_is_half_the_degree(P):
    B, H, S, D = 2, 24, 9216, 128
    _, kv = api.cpattn_exchange_bytes("kv_gather", B, H, S, D, P)
    uly_send, uly_recv = api.cpattn_exchange_bytes("ulysses", B, H, S, D, P)
    for r in range(P):
        assert kv[r] * 2 == uly_recv[r] * P          # ratio exactly P/2 for even splits
        assert uly_send[r] == uly_recv[r]


def test_closed_forms_even_split():
    B, H, S, D, P, e = 1, 8, 64, 128, 4, 2
    N = B * S * H * D * e
    send, recv = api.cpattn_exchange_bytes("ulysses", B, H, S, D, P)
    # Q, K, V and O each move (P-1)/P of the rank's N/P shard
    assert recv == [4 * (P - 1) * N // (P * P)] * P
    send, recv = api.cpattn_exchange_bytes("ring", B, H, S, D, P)
    assert recv == [2 * (P - 1) * N // P] * P       # K and V of every other chunk
    assert send == [2 * (P - 1) * N // P] * P       # own chunk to P-1 ranks
    # ring per GPU is O(n*d), Ulysses O(n*d/P): doubling P doubles the ratio
    r4 = api.cpattn_exchange_bytes("ring", B, H, S, D, 4)[1][0] / api.cpattn_exchange_bytes("ulysses", B, H, S, D, 4)[1][0]
    r8 = api.cpattn_exchange_bytes("ring", B, H, S, D, 8)[1][0] / api.cpattn_exchange_bytes("ulysses", B, H, S, D, 8)[1][0]
    assert r8 == pytest.approx(2 * r4)


def test_uneven_splits_and_degree_one():
    send, recv = api.cpattn_exchange_bytes("ulysses", 1, 30, 10007, 128, 4, [2502, 2502, 2502, 2501], [8, 8, 7, 7])
    assert sum(send) == sum(recv)                  # every byte sent is received
    s1, r1 = api.cpattn_exchange_bytes("ring", 1, 4, 100, 64, 1)
    assert s1 == [0] and r1 == [0]                 # one rank exchanges nothing
    with pytest.raises(api.CpattnError):
        api.cpattn_exchange_bytes("ulysses", 1, 30, 10007, 128, 4)   # standard mode: indivisible


# ----------------------------------------------------------------- selection model

def _pairs_brute(q0, nq, k0, nk, causal):
    return sum(sum(1 for j in range(k0, k0 + nk) if not causal or j <= i) for i in range(q0, q0 + nq))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,seq", [(16, None), (16, [5, 0, 9, 2]), (20, [1, 13, 3, 3])])
def test_plan_flops_count_visible_pairs(causal, S, seq):
    """The slowest rank's FLOPs equal 4*D*B*H times its visible (query, key)
    pairs, counted by brute force over positions."""
    B, H, D, P = 2, 3, 64, 4
    plan = api.cpattn_plan_exchange(B, H, S, D, P, 100.0, 1.0, 1000.0, causal=causal, seq_splits=seq,
                                    head_splits=[1, 1, 1, 0])
    lens = seq or [S // P] * P
    off = [0]
    for n in lens:
        off.append(off[-1] + n)
    per_rank = [sum(_pairs_brute(off[r], lens[r], off[c], lens[c], causal) for c in range(P)) for r in range(P)]
    assert plan["ring"]["flops"] == 4 * D * B * H * max(per_rank)
    uly = 4 * D * B * 1 * _pairs_brute(0, S, 0, S, causal)
    assert plan["ulysses"]["flops"] == uly
    if causal:
        assert plan["kv_gather"]["seconds"] is None and plan["best"] != "kv_gather"
    else:
        assert plan["kv_gather"]["flops"] == plan["ring"]["flops"]


def test_plan_times_by_hand():
    """P = 2, equal shards of 4 tokens, B = H = 1, D = 16, bf16; link 1 GB/s,
    1 TFLOP/s, HBM 2 GB/s."""
    B, H, S, D, P = 1, 2, 8, 16, 2
    plan = api.cpattn_plan_exchange(B, H, S, D, P, 1.0, 1.0, 2.0)
    row = D * 2
    a = 4 * D * B * H * 16 / 1e12                       # one shard against one chunk: 4 x 4 pairs, 2 heads
    hop = 2 * B * 4 * H * row / 1e9                     # K and V of one chunk
    assert plan["ring"]["seconds"] == pytest.approx(a + max(a, hop), rel=1e-12)
    recv_kv = 2 * B * 4 * H * row                       # the other chunk's K and V
    assert plan["kv_gather"]["seconds"] == pytest.approx(recv_kv / 1e9 + 2 * a, rel=1e-12)
    recv_u = (3 * B * 4 * 1 + B * 4 * 1) * row          # 3 tensors in for 1 head of 4 tokens, O back
    t_u = recv_u / 1e9 + 8 * B * 4 * H * row / 2e9 + 4 * D * B * 1 * 64 / 1e12
    assert plan["ulysses"]["seconds"] == pytest.approx(t_u, rel=1e-12)
    assert plan["ring"]["resident_bytes"] == (2 * 4 + 4 * 4) * B * H * row
    assert plan["ulysses"]["resident_bytes"] == 4 * B * S * 1 * row
    assert plan["kv_gather"]["resident_bytes"] == (2 * 4 + 2 * S) * B * H * row


def test_plan_limits_follow_the_pages():
    B, H, S, D = 1, 24, 4608, 128
    # a fast link: communication vanishes, ring and kv_gather cost the same compute
    fast = api.cpattn_plan_exchange(B, H, S, D, 4, 1e12, 1000.0, 6000.0)
    assert fast["ring"]["seconds"] == pytest.approx(fast["kv_gather"]["seconds"], rel=1e-6)
    assert fast["best"] in ("ring", "kv_gather")
    # a slow link: payload decides; Ulysses moves the least for P >= 4 ([USP] section 5)
    for P in (4, 8):
        slow = api.cpattn_plan_exchange(B, H, S, D, P, 1.0, 1000.0, 6000.0)
        assert slow["best"] == "ulysses"
        assert slow["kv_gather"]["recv_bytes"] * 2 == slow["ulysses"]["recv_bytes"] * P
    # SP2: the kv_gather and Ulysses payloads are about equal
    sp2 = api.cpattn_plan_exchange(B, H, S, D, 2, 1.0, 1000.0, 6000.0)
    assert sp2["kv_gather"]["recv_bytes"] == sp2["ulysses"]["recv_bytes"]
    # Ulysses holds less attention activation memory than kv_gather
    for P in (2, 4, 8):
        pl = api.cpattn_plan_exchange(B, H, S, D, P, 770.0, 1000.0, 6000.0)
        assert pl["ulysses"]["resident_bytes"] < pl["kv_gather"]["resident_bytes"]


def test_plan_feasibility_and_validation():
    lib = api._native.load()
    # heads not divisible and no splits: Ulysses is infeasible, the others are not
    pl = api.cpattn_plan_exchange(1, 30, 4096, 128, 4, 770.0, 1000.0, 6000.0)
    assert pl["ulysses"]["seconds"] is None and pl["best"] in ("ring", "kv_gather")
    # with explicit head splits it is feasible again (Ulysses Anything)
    pl = api.cpattn_plan_exchange(1, 30, 4096, 128, 4, 770.0, 1000.0, 6000.0, head_splits=[8, 8, 7, 7])
    assert pl["ulysses"]["seconds"] is not None
    env = api._ExchangeEnv(770.0, 1000.0, 6000.0, 0)
    plan = api._ExchangePlan()
    import ctypes
    assert lib.cpattn_plan_exchange(1, 4, 8, 64, 2, 2, None, None, None, ctypes.byref(plan)) == 1        # NULL
    assert lib.cpattn_plan_exchange(1, 4, 8, 64, 2, 2, None, None, ctypes.byref(env), None) == 1
    bad = api._ExchangeEnv(0.0, 1000.0, 6000.0, 0)
    assert lib.cpattn_plan_exchange(1, 4, 8, 64, 2, 2, None, None, ctypes.byref(bad), ctypes.byref(plan)) == 2
    assert lib.cpattn_plan_exchange(1, 4, 9, 64, 2, 2, None, None, ctypes.byref(env), ctypes.byref(plan)) == 3
    assert lib.cpattn_plan_exchange(1, 4, 8, 64, 2, 0, None, None, ctypes.byref(env), ctypes.byref(plan)) == 5
    bad_heads = api._native.int_array([3, 3])
    assert lib.cpattn_plan_exchange(1, 4, 8, 64, 2, 2, None, bad_heads, ctypes.byref(env), ctypes.byref(plan)) == 4
