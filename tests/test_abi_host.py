"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, and validates shapes and capacities."""

import ctypes

import pytest
import torch

import block_sparse_attention_star_b200 as star
from synth import CONFIGS


def test_library_exports_every_header_symbol():
    lib = star.lib()
    syms = star.header_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(lib, s), s
    assert star.star_version().startswith("star-b200")


def _shape(**kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, L=131072, b=32768, T_max=128)
    base.update(kw)
    return star.StarShape.make(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(L=131000), star.STAR_ERR_UNSUPPORTED_SHAPE),          # ragged last block
    (dict(Hq=24, Hkv=8), star.STAR_ERR_UNSUPPORTED_SHAPE),      # group of 3
    (dict(Hq=30, Hkv=8), star.STAR_ERR_INVALID_ARG),            # not a multiple
    (dict(d=96), star.STAR_ERR_UNSUPPORTED_SHAPE),
    (dict(b=32704, L=32704 * 4), star.STAR_ERR_UNSUPPORTED_SHAPE),  # b not a multiple of 128
    (dict(B=0), star.STAR_ERR_INVALID_ARG),
    (dict(rope_theta=-1.0), star.STAR_ERR_INVALID_ARG),
    (dict(anchor=-128), star.STAR_ERR_INVALID_ARG),              # negative anchor size
    (dict(anchor=1000), star.STAR_ERR_UNSUPPORTED_SHAPE),         # anchor not a multiple of 128
    (dict(anchor=32768 + 128), star.STAR_ERR_UNSUPPORTED_SHAPE),  # anchor larger than the block
    (dict(B=2, seq_len=(0, 131072)), star.STAR_ERR_INVALID_ARG),   # an empty context
    (dict(seq_len=(131072 + 1,)), star.STAR_ERR_INVALID_ARG),      # longer than the capacity L
])
def test_shape_validation(kw, code):
    with pytest.raises(star.StarError) as e:
        star.star_pages_needed(_shape(**kw))
    assert e.value.code == code
    assert star.lib().star_last_error().decode()


def test_pages_and_page_table():
    sh = _shape()
    need = star.star_pages_needed(sh)
    assert need == (131072 + 128 + 255) // 256
    tab = star.star_page_table_fill(sh, need, first_page=5)
    assert tab.shape == (1, need) and tab[0, 0] == 5 and tab[0, -1] == 5 + need - 1
    with pytest.raises(star.StarError) as e:
        star.star_page_table_fill(sh, need - 1)
    assert e.value.code == star.STAR_ERR_CAPACITY


def test_workspace_sizes_for_every_workload():
    for wl in CONFIGS.values():
        sh = star.StarShape.make(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, L=wl.L, b=wl.b, T_max=wl.T_max)
        assert star.star_workspace_size(sh, star.STAR_OP_PHASE1) == 0
        ws2 = star.star_workspace_size(sh, star.STAR_OP_PHASE2, wl.T)
        wsd = star.star_workspace_size(sh, star.STAR_OP_DECODE)
        assert ws2 % 256 == 0 and wsd % 256 == 0 and wsd > 0
        with pytest.raises(star.StarError):
            star.star_workspace_size(sh, star.STAR_OP_PHASE2, wl.T_max + 1)


def test_bench_shape_carries_every_workload_field():
    """The timed shape is the workload's: anchor and per-sequence context lengths included."""
    import bench
    for wl in CONFIGS.values():
        sh = bench.workload_shape(wl)
        assert (sh.B, sh.Hq, sh.Hkv, sh.d, sh.L, sh.b, sh.T_max) == (wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.b, wl.T_max)
        assert sh.anchor == (wl.anchor or 0)
        if wl.seq_lens is None:
            assert not sh.seq_len
        else:
            assert [sh.seq_len[i] for i in range(wl.B)] == list(wl.seq_lens)


def test_anchor_workspace_size():
    """The anchor's keys roped at caller ids: bf16 [B][n-1][Hkv][a][d]; a = b when the shape says 0."""
    for a in (0, 8192, 32768):
        sh = _shape(B=2, anchor=a)
        aa = a or 32768
        assert star.star_workspace_size(sh, star.STAR_OP_PHASE1_ANCHOR) == 2 * 3 * 8 * aa * 128 * 2
    one_block = _shape(L=32768, b=32768)
    assert star.star_workspace_size(one_block, star.STAR_OP_PHASE1_ANCHOR) == 0


def test_null_arguments_rejected_before_any_launch():
    lib = star.lib()
    sh = _shape()
    rc = lib.star_phase1_encode(ctypes.byref(sh), None, None, None, None, None, None, None, 0, None)
    assert rc == star.STAR_ERR_INVALID_ARG
    rc = lib.star_lse_merge(0, 10, 128, None, None, None, None, None)
    assert rc == star.STAR_ERR_INVALID_ARG
    rc = lib.star_lse_merge(2, 10, 96, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), None, None)
    assert rc == star.STAR_ERR_UNSUPPORTED_SHAPE
    rc = lib.star_set_trace_events(ctypes.c_void_p(16), None)
    assert rc == star.STAR_ERR_INVALID_ARG


def test_phase2_and_decode_workspaces_are_checked_before_any_launch():
    """Phase 2 always needs its workspace (RoPE(q) is staged there); both calls check its size."""
    lib = star.lib()
    sh = _shape()
    max_pages = ctypes.c_int32()
    assert lib.star_pages_needed(ctypes.byref(sh), ctypes.byref(max_pages)) == star.STAR_OK
    # Never dereferenced: every call below fails its argument checks first.
    cache = star.StarCache(k_pool=256, v_pool=256, page_table=256, max_pages=max_pages.value, num_pages=1)
    p = ctypes.c_void_p(256)
    T = 64
    need = star.star_workspace_size(sh, star.STAR_OP_PHASE2, T)
    assert need >= sh.B * T * sh.Hq * sh.d * 2
    rc = lib.star_phase2_partial(ctypes.byref(sh), ctypes.byref(cache), p, None, None, p, T, p, p, None, 0, None)
    assert rc == star.STAR_ERR_INVALID_ARG  # ws is NULL
    rc = lib.star_phase2_partial(ctypes.byref(sh), ctypes.byref(cache), p, None, None, p, T, p, p, p, need - 256, None)
    assert rc == star.STAR_ERR_CAPACITY
    need_d = star.star_workspace_size(sh, star.STAR_OP_DECODE)
    rc = lib.star_decode_step(ctypes.byref(sh), ctypes.byref(cache), p, p, p, p, sh.L, p, None, p, need_d - 256,
                              None)
    assert rc == star.STAR_ERR_CAPACITY


def test_encode_layers_callback_marshalling_without_a_launch():
    """star_encode_layers validates its arguments, then calls the caller's callback before
    any launch: an exception raised there stops the call (STAR_ERR_CALLBACK in C) and is
    raised again by the binding, with no CUDA call made."""
    sh = _shape(L=512, b=256)
    max_pages = star.star_pages_needed(sh)

    class FakeCache:  # never dereferenced: the call stops in the first callback
        c = star.StarCache(k_pool=256, v_pool=256, page_table=256, max_pages=max_pages, num_pages=1)

    x = torch.zeros(16, dtype=torch.bfloat16)
    t = torch.zeros(16, dtype=torch.bfloat16)
    pos = torch.zeros(16, dtype=torch.int32)
    calls = []

    def fn(layer, stage, *tensors):
        calls.append((layer, stage, len(tensors)))
        raise KeyError("model failed")

    with pytest.raises(KeyError):
        star.star_encode_layers(sh, [FakeCache(), FakeCache()], pos, x, t, t, t, t, fn, stream=0)
    assert calls == [(0, star.STAR_LAYER_QKV, 5)]
    assert "callback" in star.lib().star_last_error().decode()
    with pytest.raises(star.StarError) as e:  # a NULL callback is rejected up front
        star._check(star.lib().star_encode_layers(ctypes.byref(sh), 1, ctypes.byref(FakeCache.c), None, None, None,
                                                  None, None, None, star.LAYER_FN(), None, None))
    assert e.value.code == star.STAR_ERR_INVALID_ARG


def test_exchange_buffer_size_and_checks():
    """The peer-exchange buffer: a 256-byte header, then 2 parities x world slots of
    slots x rows partials (f32 O rows of d, then f32 LSEs), each part rounded up to 256 bytes."""
    import block_sparse_attention_star_b200 as star
    def rup(x):
        return (x + 255) // 256 * 256
    for world, slots, rows, d in [(1, 4, 2048, 128), (2, 2, 2048, 128), (8, 1, 32, 128), (3, 5, 7, 64)]:
        slot = rup(slots * rows * d * 4) + rup(slots * rows * 4)
        assert star.star_exchange_size(world, slots, rows, d) == 256 + 2 * world * slot
    for bad, code in [((9, 1, 32, 128), star.STAR_ERR_UNSUPPORTED_SHAPE), ((2, 0, 32, 128), star.STAR_ERR_INVALID_ARG),
                      ((2, 1, 32, 96), star.STAR_ERR_UNSUPPORTED_SHAPE)]:
        with pytest.raises(star.StarError) as e:
            star.star_exchange_size(*bad)
        assert e.value.code == code


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without libstar.so every call raises instead of computing anything."""
    monkeypatch.setattr(star, "_lib", None)
    monkeypatch.setattr(star, "LIB_PATH", str(tmp_path / "libstar.so"))
    with pytest.raises(ImportError, match="missing"):
        star.star_version()
    with pytest.raises(ImportError, match="missing"):
        star.star_lse_merge(1, 1, 128, torch.zeros(1, 1, 128), torch.zeros(1, 1), torch.zeros(1, 128),
                            torch.zeros(1))
