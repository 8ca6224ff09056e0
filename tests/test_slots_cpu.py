"""Slot-indexed state pools, host side (no GPU): the indexed entry points
refuse bad slot arguments before touching any buffer, and the indexed
prefill's workspace is gdn_prefill's plus one state and one conv-history
buffer per sequence."""

import numpy as np
import pytest

import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi


@pytest.fixture(scope="module", autouse=True)
def built():
    from linear_attention_recurrence_deltanet_b200 import build
    build.build()
    yield


class FakeTensor:
    """Host memory standing in for a device tensor: validation must reject the
    call before anything reads or writes it."""

    def __init__(self, nbytes, offset=0):
        self.view = np.arange(nbytes + 64, dtype=np.uint8)
        self.offset = offset

    def data_ptr(self):
        return self.view.ctypes.data + self.offset

    def numel(self):
        return self.view.size

    def element_size(self):
        return 1


def bufs(geo, N, slots, K=1, T=None):
    T = N * K if T is None else T
    io = geo.io_bytes
    t = dict(qkv=FakeTensor(T * geo.conv_dim * io), z=FakeTensor(T * geo.value_dim * io),
             a=FakeTensor(T * geo.num_v_heads * io), b=FakeTensor(T * geo.num_v_heads * io),
             conv=FakeTensor(slots * 3 * geo.conv_dim * io), idx=FakeTensor(4 * N),
             state=FakeTensor(slots * geo.num_v_heads * geo.head_v_dim * geo.head_k_dim * 4),
             o=FakeTensor(T * geo.value_dim * io), ws=FakeTensor(1 << 12))
    params = tuple(FakeTensor(n) for n in (geo.conv_dim * 16, 4 * geo.num_v_heads, 4 * geo.num_v_heads,
                                           4 * geo.head_v_dim))
    return t, params


def test_indexed_decode_rejects_bad_slot_arguments():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6)
    cfg = gdn.make_config(geo)
    t, params = bufs(geo, 2, 4, K=2)
    snap = {k: v.view.copy() for k, v in t.items()}
    bad_idx = FakeTensor(8, offset=2)
    cases = [
        (dict(idx=None, slots=4), "GDN_E_INVAL"),       # no slot array
        (dict(idx=t["idx"], slots=0), "GDN_E_INVAL"),   # empty pool
        (dict(idx=t["idx"], slots=70000), "GDN_E_INVAL"),
        (dict(idx=bad_idx, slots=4), "GDN_E_INVAL"),    # misaligned slot array
    ]
    for kw, status in cases:
        with pytest.raises(gdn.GdnError) as e:
            gdn.decode_step_indexed(cfg, params, t["qkv"], t["z"], t["a"], t["b"], 2, kw["idx"], kw["slots"],
                                    t["conv"], t["state"], t["o"], stream=0)
        assert e.value.name == status, kw
        with pytest.raises(gdn.GdnError) as e:
            gdn.decode_multi_indexed(cfg, params, t["qkv"], t["z"], t["a"], t["b"], 2, 2, True, None, kw["idx"],
                                     kw["slots"], t["conv"], t["state"], t["o"], stream=0)
        assert e.value.name == status, kw
    # the unindexed checks still apply to the indexed calls
    with pytest.raises(gdn.GdnError) as e:
        gdn.decode_multi_indexed(cfg, params, t["qkv"], t["z"], t["a"], t["b"], 2, 5, True, None, t["idx"], 4,
                                 t["conv"], t["state"], t["o"], stream=0)
    assert e.value.name == "GDN_E_INVAL"
    with pytest.raises(gdn.GdnError) as e:
        gdn.decode_step_indexed(cfg, params, t["qkv"], t["z"], t["a"], t["b"], 0, t["idx"], 4, t["conv"],
                                t["state"], t["o"], stream=0)
    assert e.value.name == "GDN_E_INVAL"
    for k, v in t.items():
        assert np.array_equal(v.view, snap[k]), k


def test_indexed_prefill_workspace_adds_one_state_and_history_per_sequence():
    geo = gi.Geometry()
    cfg = gdn.make_config(geo)
    per_seq = geo.num_v_heads * geo.head_v_dim * geo.head_k_dim * 4 + 3 * geo.conv_dim * geo.io_bytes
    for T, N, chunk in [(4096, 1, 64), (65536, 16, 64), (1000, 7, 16), (300, 3, 128)]:
        base = gdn.prefill_workspace_size(cfg, T, N, chunk)
        full = gdn.prefill_indexed_workspace_size(cfg, T, N, chunk)
        assert base + N * per_seq <= full <= base + N * per_seq + 3 * 256, (T, N, chunk)


def test_indexed_prefill_rejects_before_launch():
    geo = gi.Geometry()
    cfg = gdn.make_config(geo)
    t, params = bufs(geo, 2, 3, T=16)
    cu_dev = FakeTensor(12)
    snap = {k: v.view.copy() for k, v in t.items()}

    def call(idx=t["idx"], slots=3, cu_host=(0, 9, 16), chunk=64, flags=0, wsb=None):
        gdn.prefill_indexed(cfg, params, t["qkv"], t["z"], t["a"], t["b"], cu_dev, list(cu_host), idx, slots, chunk,
                            flags, t["conv"], t["state"], t["o"], t["ws"], workspace_bytes=wsb, stream=0)

    need = gdn.prefill_indexed_workspace_size(cfg, 16, 2, 64)
    cases = [
        (dict(idx=None), "GDN_E_INVAL"),
        (dict(slots=0), "GDN_E_INVAL"),
        (dict(cu_host=(0, 9, 4)), "GDN_E_INVAL"),
        (dict(chunk=48), "GDN_E_INVAL"),
        (dict(flags=0x40), "GDN_E_INVAL"),
        (dict(wsb=need - 256), "GDN_E_WORKSPACE"),   # room for gdn_prefill but not for the slot buffers
    ]
    for kw, status in cases:
        with pytest.raises(gdn.GdnError) as e:
            call(**kw)
        assert e.value.name == status, (kw, e.value)
    for k, v in t.items():
        assert np.array_equal(v.view, snap[k]), k
