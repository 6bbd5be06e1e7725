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
