"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects invalid arguments with the documented status codes
before touching CUDA.  Pointers passed here are fake (never dereferenced):
every call below must fail validation."""
import ctypes
import os
import re

import pytest
import torch

from context_attention_long_b200 import _native, build, inputs

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "cpattn.h")

OK, NULL, SHAPE, INDIV, SPLITS, DEGREE, CUDA, TIMEOUT, WS, ALIGN, UNSUP = range(11)
FAKE = ctypes.c_void_p(1 << 20)      # non-null, 16-byte aligned, never dereferenced
FAKE_MIS = ctypes.c_void_p((1 << 20) + 8)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cpattn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for required in ("cpattn_ring_attention", "cpattn_lse_merge", "cpattn_ulysses_permute",
                     "cpattn_ulysses_unpermute", "cpattn_kv_gather_attention"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name
        assert name in _native.SIGNATURES, f"{name} has no ctypes signature"


def test_status_strings(lib):
    for code in range(11):
        s = lib.cpattn_status_string(code).decode()
        assert s.startswith("CPATTN")
    assert b"unknown" in lib.cpattn_status_string(99)
    assert lib.cpattn_version() >= 10000


def test_front_loaded_splits_agree_with_input_recipe(lib):
    for total, parts in [(30, 4), (10007, 4), (4095, 2), (7, 7), (5, 8), (0, 3), (4608, 4)]:
        arr = (ctypes.c_int * parts)()
        assert lib.cpattn_front_loaded_splits(total, parts, arr) == OK
        assert list(arr) == inputs.front_loaded_splits(total, parts)
    assert lib.cpattn_front_loaded_splits(5, 0, (ctypes.c_int * 1)()) == DEGREE
    assert lib.cpattn_front_loaded_splits(5, 2, None) == NULL


def _ring(lib, q=FAKE, out=FAKE, B=1, H=2, S=256, D=64, P=4, lens=None, lse=FAKE):
    return lib.cpattn_ring_attention(q, FAKE, FAKE, out, lse, B, H, S, D, P, _native.int_array(lens), None)


def test_ring_validation(lib):
    assert _ring(lib, q=None) == NULL
    assert _ring(lib, out=None) == NULL
    assert _ring(lib, D=96) == SHAPE
    assert _ring(lib, B=0) == SHAPE
    assert _ring(lib, S=0) == SHAPE
    assert _ring(lib, P=0) == DEGREE
    assert _ring(lib, S=10, P=3) == INDIV                    # standard ring: S % ring_degree != 0
    assert _ring(lib, S=3, P=4) == DEGREE                    # more ranks than tokens, equal split
    assert _ring(lib, S=10, P=3, lens=[3, 3, 3]) == SPLITS   # Ring Anything lengths must sum to S
    assert _ring(lib, S=10, P=3, lens=[11, -1, 0]) == SPLITS
    assert _ring(lib, q=FAKE_MIS) == ALIGN


def test_ring_step_validation(lib):
    f = lambda step, lse=FAKE: lib.cpattn_ring_step(FAKE, FAKE, FAKE, FAKE, lse, 1, 2, 256, 64, 4, None, step, None)
    assert f(-1) == DEGREE
    assert f(4) == DEGREE
    assert f(0, lse=None) == NULL


def test_merge_validation(lib):
    f = lambda **kw: lib.cpattn_lse_merge(kw.get("po", FAKE), kw.get("pl", FAKE), kw.get("P", 4), 1, 2, 8,
                                          kw.get("D", 64), kw.get("of", FAKE), kw.get("ob", None), FAKE, None)
    assert f(po=None) == NULL
    assert f(of=None, ob=None) == NULL
    assert f(P=0) == SHAPE
    assert f(D=32) == SHAPE
    assert f(po=FAKE_MIS) == ALIGN


def test_kv_gather_validation(lib):
    f = lambda S=16, P=4, lens=None: lib.cpattn_kv_gather_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, S, 64, P,
                                                                    _native.int_array(lens), None)
    assert f(S=18) == INDIV
    assert f(lens=[4, 4, 4, 5]) == SPLITS
    assert f(P=0) == DEGREE


def test_permute_validation(lib):
    def f(x=FAKE, y=FAKE, B=1, S=8, H=4, D=64, eb=2, P=2, seq=None, heads=None):
        return lib.cpattn_ulysses_permute(x, y, B, S, H, D, eb, P, _native.int_array(seq), _native.int_array(heads), None)
    assert f(x=None) == NULL
    assert f(eb=3) == SHAPE
    assert f(D=3, eb=2) == SHAPE        # rows must be a multiple of 16 bytes
    assert f(P=0) == DEGREE
    assert f(H=5) == INDIV              # standard Ulysses: heads % degree != 0
    assert f(S=9) == INDIV              # standard Ulysses: seq % degree != 0
    assert f(H=5, heads=[3, 3]) == SPLITS
    assert f(S=9, seq=[5, 5]) == SPLITS
    assert f(y=FAKE_MIS) == ALIGN
    g = lambda H=5: lib.cpattn_ulysses_unpermute(FAKE, FAKE, 1, 8, H, 64, 2, 2, None, None, None)
    assert g() == INDIV
    t = lambda k=FAKE, yv=FAKE, H=4: lib.cpattn_ulysses_permute_qkv(FAKE, k, FAKE, FAKE, FAKE, yv, 1, 8, H, 64, 2, 2,
                                                                    None, None, None)
    assert t(k=None) == NULL
    assert t(yv=FAKE_MIS) == ALIGN
    assert t(H=5) == INDIV


def test_projection_validation(lib):
    def q(x=FAKE, w=FAKE, yq=FAKE, yv=FAKE, B=1, S=8, H=4, D=64, Dm=128, P=2, seq=None, heads=None):
        return lib.cpattn_ulysses_qkv_projection(x, w, yq, FAKE, yv, B, S, H, D, Dm, P, _native.int_array(seq),
                                                 _native.int_array(heads), None)
    assert q(x=None) == NULL
    assert q(w=None) == NULL
    assert q(yv=None) == NULL
    assert q(D=32) == SHAPE
    assert q(Dm=96) == SHAPE            # Dm must be a multiple of 64
    assert q(Dm=0) == SHAPE
    assert q(B=0) == SHAPE
    assert q(H=2000) == SHAPE
    assert q(S=1 << 29, H=1024, D=128) == SHAPE   # within every other bound, but more 256 x 256 tiles than an int numbers
    assert q(P=0) == DEGREE
    assert q(P=65) == DEGREE
    assert q(H=5) == INDIV
    assert q(S=9, seq=[5, 5]) == SPLITS
    assert q(H=5, heads=[4, 2]) == SPLITS
    assert q(x=FAKE_MIS) == ALIGN
    assert q(yq=FAKE_MIS) == ALIGN

    def o(yo=FAKE, w=FAKE, out=FAKE, H=4, D=64, Dm=128, P=2):
        return lib.cpattn_ulysses_output_projection(yo, w, out, 1, 8, H, D, Dm, P, None, None, None)
    assert o(out=None) == NULL
    assert o(yo=None) == NULL
    assert o(Dm=100) == SHAPE
    assert o(D=96) == SHAPE
    assert o(H=5) == INDIV
    assert o(out=FAKE_MIS) == ALIGN
    assert o(w=FAKE_MIS) == ALIGN


def test_flow_validation(lib):
    need = lib.cpattn_ulysses_workspace_bytes(1, 4, 8, 64)
    assert need == 4 * 1 * 8 * 4 * 64 * 2
    assert lib.cpattn_unified_workspace_bytes(1, 4, 8, 64) == need
    u = lambda ws=FAKE, nbytes=need, H=4: lib.cpattn_ulysses_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, H, 8, 64, 2,
                                                                       None, None, ws, nbytes, None)
    assert u(ws=None) == WS
    assert u(nbytes=need - 1) == WS
    assert u(H=5) == INDIV
    v = lambda ws=FAKE, R=2, U=2: lib.cpattn_unified_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 8, 64, R, U, None,
                                                               None, ws, need, None)
    assert v(ws=None) == WS
    assert v(R=3) == INDIV
    assert v(U=3) == INDIV
    assert v(R=0) == DEGREE
    h = lambda H=4: lib.cpattn_head_sharded_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, H, 8, 64, 2, None, None)
    assert h(H=5) == INDIV


def test_noalloc_validation(lib):
    # Every case returns before the library touches CUDA (the scratch-size
    # check comes before the device check), so these run without a GPU.
    def f(q=FAKE, out=FAKE, B=1, S=8, H=4, D=64, P=2, seq=None, heads=None):
        return lib.cpattn_ulysses_attention_noalloc(q, FAKE, FAKE, out, FAKE, B, H, S, D, P, _native.int_array(seq),
                                                    _native.int_array(heads), None)
    assert f(q=None) == NULL
    assert f(out=None) == NULL
    assert f(D=96) == SHAPE
    assert f(P=0) == DEGREE
    assert f(P=65) == DEGREE
    assert f(H=5) == INDIV
    assert f(S=9) == INDIV
    assert f(S=9, seq=[5, 5]) == SPLITS
    assert f(H=5, heads=[3, 3]) == SPLITS
    assert f(seq=[9, -1]) == SPLITS
    # 8 * B*S*H*D bytes of scratch against the 64 MiB array: 1 x 8192 x 8 x 128
    # fills it exactly, one more token does not fit.
    assert f(S=8193, H=8, D=128, P=1) == WS
    assert f(B=2, S=4097, H=8, D=128, P=1) == WS


def test_debug_hook_validation(lib):
    assert lib.cpattn_debug_wait_timeout(0, None) == SHAPE
    assert lib.cpattn_device_status(None, None) == NULL


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_gpu_reports_cuda_error(lib):
    # Arguments pass validation; with no device the call must return
    # CPATTN_ERR_CUDA before launching anything, and record on this thread
    # which CUDA call failed and why.
    assert _ring(lib) == CUDA
    assert lib.cpattn_last_cuda_error() != 0
    assert lib.cpattn_last_cuda_error_string().decode().startswith("device query: cudaError")


def test_last_cuda_error_is_thread_local(lib):
    import threading
    seen = []
    t = threading.Thread(target=lambda: seen.append((lib.cpattn_last_cuda_error(),
                                                     lib.cpattn_last_cuda_error_string().decode())))
    t.start()
    t.join()
    assert seen == [(0, "no CUDA error recorded on this thread")]


def test_causal_entry_points_validate_like_their_namesakes(lib):
    r = lambda q=FAKE, S=256, P=4, lens=None: lib.cpattn_causal_ring_attention(q, FAKE, FAKE, FAKE, FAKE, 1, 2, S, 64,
                                                                              P, _native.int_array(lens), None)
    assert r(q=None) == NULL
    assert r(S=10, P=3) == INDIV
    assert r(S=10, P=3, lens=[3, 3, 3]) == SPLITS
    assert r(q=FAKE_MIS) == ALIGN
    st = lambda step, lse=FAKE: lib.cpattn_causal_ring_step(FAKE, FAKE, FAKE, FAKE, lse, 1, 2, 256, 64, 4, None,
                                                             step, None)
    assert st(-1) == DEGREE and st(4) == DEGREE and st(0, lse=None) == NULL
    h = lambda H=4: lib.cpattn_causal_head_sharded_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, H, 8, 64, 2, None, None)
    assert h(H=5) == INDIV
    need = lib.cpattn_ulysses_workspace_bytes(1, 4, 8, 64)
    u = lambda ws=FAKE, H=4: lib.cpattn_causal_ulysses_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, H, 8, 64, 2, None,
                                                                 None, ws, need, None)
    assert u(ws=None) == WS and u(H=5) == INDIV
    v = lambda ws=FAKE, R=2: lib.cpattn_causal_unified_attention(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 8, 64, R, 2,
                                                                 None, None, ws, need, None)
    assert v(ws=None) == WS and v(R=3) == INDIV
    if not torch.cuda.is_available():
        assert r() == CUDA       # valid arguments, no device: fails before any launch


def test_backward_validation(lib):
    need = lib.cpattn_attention_backward_workspace_bytes(1, 2, 256)
    assert need == 1 * 2 * 256 * 4
    assert lib.cpattn_attention_backward_workspace_bytes(0, 2, 256) == 0

    def f(q=FAKE, lse=FAKE, dq=FAKE, D=64, S=256, ws=FAKE, nbytes=need):
        return lib.cpattn_attention_backward(q, FAKE, FAKE, FAKE, lse, FAKE, dq, FAKE, FAKE, 1, 2, S, D, 1, ws,
                                             nbytes, None)
    assert f(q=None) == NULL
    assert f(lse=None) == NULL
    assert f(D=96) == SHAPE
    assert f(S=0) == SHAPE
    # B*S*H >= 2^31 (here 2 heads x 2^30 tokens): rows are indexed in 32 bits
    assert f(S=1 << 30, nbytes=1 << 40) == SHAPE
    assert f(ws=None) == WS
    assert f(nbytes=need - 4) == WS
    assert f(dq=FAKE_MIS) == ALIGN
    if not torch.cuda.is_available():
        assert f() == CUDA


def test_backward_ds_bytes(lib):
    """dS scratch per head: B x 32 KB (a 128 x 128 bf16 tile) per (Q tile, K
    tile) pair the dK/dV kernel walks -- every pair, or under the causal mask
    the pairs whose K tile starts at or before the Q tile's last query
    (counted here by brute force)."""
    for B, S in ((1, 1), (2, 300), (1, 4608), (3, 257), (1, 9216)):
        nt = (S + 127) // 128
        causal_pairs = sum(1 for qt in range(nt) for kt in range(nt) if kt * 128 <= min(S, qt * 128 + 128) - 1)
        assert lib.cpattn_attention_backward_ds_bytes(B, S, 0) == B * nt * nt * 128 * 128 * 2
        assert lib.cpattn_attention_backward_ds_bytes(B, S, 1) == B * causal_pairs * 128 * 128 * 2
    assert lib.cpattn_attention_backward_ds_bytes(1, 4608, 0) == 42467328     # image-DiT: 42.5 MB per head
    assert lib.cpattn_attention_backward_ds_bytes(0, 256, 0) == 0
    assert lib.cpattn_attention_backward_ds_bytes(1, 0, 1) == 0


def test_backward_workspace_budget():
    """The bindings add whole heads of dS scratch within the budget (plus
    256 bytes of alignment slack), or none when one head does not fit."""
    from context_attention_long_b200 import api
    base = api.cpattn_attention_backward_workspace_bytes(2, 5, 300)
    per = api.cpattn_attention_backward_ds_bytes(2, 300, False)
    assert api.backward_workspace_bytes(2, 5, 300) == base + 256 + 5 * per
    assert api.backward_workspace_bytes(2, 5, 300, ds_budget=0) == base
    assert api.backward_workspace_bytes(2, 5, 300, ds_budget=per - 1) == base
    assert api.backward_workspace_bytes(2, 5, 300, ds_budget=2 * per + 7) == base + 256 + 2 * per
    per_c = api.cpattn_attention_backward_ds_bytes(2, 300, True)
    assert api.backward_workspace_bytes(2, 5, 300, causal=True, ds_budget=2 * per) == base + 256 + 3 * per_c
    ubase = api.cpattn_ulysses_attention_backward_workspace_bytes(2, 5, 300, 64)
    assert api.backward_workspace_bytes(2, 5, 300, ulysses_D=64, ds_budget=per) == ubase + 256 + per
    # the video workload: 2 GiB of dS per head, so the default budget takes 4 of its 40 heads
    per_v = api.cpattn_attention_backward_ds_bytes(1, 32760, False)
    assert per_v == 256 * 256 * 32768
    assert api.backward_workspace_bytes(1, 40, 32760) == (api.cpattn_attention_backward_workspace_bytes(1, 40, 32760)
                                                          + 256 + (api.BACKWARD_DS_BUDGET // per_v) * per_v)


def test_ulysses_backward_validation(lib):
    need = lib.cpattn_ulysses_attention_backward_workspace_bytes(1, 4, 8, 64)
    assert need == 10 * 1 * 8 * 4 * 64 + 4 * 1 * 4 * 8

    def f(ws=FAKE, nbytes=need, H=4, heads=None, lse=FAKE):
        return lib.cpattn_ulysses_attention_backward(FAKE, FAKE, FAKE, FAKE, lse, FAKE, FAKE, FAKE, FAKE, 1, H, 8,
                                                     64, 2, None, _native.int_array(heads), 0, ws, nbytes, None)
    assert f(lse=None) == NULL
    assert f(ws=None) == WS
    assert f(nbytes=need - 1) == WS
    assert f(H=5) == INDIV
    assert f(heads=[3, 3]) == SPLITS
    assert f(ws=FAKE_MIS) == ALIGN


def test_binding_refuses_host_and_strided_tensors():
    """Host tensors never reach the library as pointers (they would be device
    addresses to the kernels); the check runs before any library call."""
    from context_attention_long_b200 import api
    x = torch.zeros(2 * 8 * 4 * 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.cpattn_ulysses_permute(x, 2, 8, 4, 64, 2, y=torch.empty_like(x))
    with pytest.raises(ValueError):
        api._ptr(torch.zeros(4, 4).t())      # a CPU, non-contiguous view
    assert api._ptr(None) is None


def test_binding_refuses_short_or_mistyped_buffers():
    """A buffer smaller than the sizes passed, or of the wrong dtype, is refused
    before the library would index past it."""
    from context_attention_long_b200 import api
    with pytest.raises(ValueError):
        api._need(torch.zeros(10, dtype=torch.bfloat16), 11, torch.bfloat16, "x")
    with pytest.raises(ValueError):
        api._need(torch.zeros(10, dtype=torch.float32), 10, torch.bfloat16, "x")
    api._need(torch.zeros(12, dtype=torch.bfloat16), 11, torch.bfloat16, "x")
    api._need(None, 11, torch.bfloat16, "x")
    x = torch.zeros(2 * 8 * 4 * 64 - 1, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.cpattn_ulysses_permute(x, 2, 8, 4, 64, 2)
