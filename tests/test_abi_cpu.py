"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments and bad state blobs on the host
before touching any buffer."""

import ctypes
import os
import re
import struct

import numpy as np
import pytest

import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from linear_attention_recurrence_deltanet_b200 import build
    build.build()
    yield


def header_functions():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    L = gdn.lib()
    declared = header_functions()
    assert len(declared) >= 17
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(gdn.EXPORTS) == declared


def test_debug_wait_expiry_limit_validated_on_the_host():
    for bad in (0, 1000001):
        with pytest.raises(gdn.GdnError) as e:
            gdn.debug_wait_expiry(bad, stream=0)
        assert e.value.name == "GDN_E_INVAL" and "limit_us" in str(e.value)


def test_abi_version_and_names():
    assert gdn.abi_version() == 1
    assert gdn.kernel_name(gdn.K.DECODE) == "decode"
    assert gdn.kernel_name(99) == "unknown"


def qwen_cfg(**kw):
    return gdn.make_config(gi.Geometry(**kw))


@pytest.mark.parametrize("kw,status", [
    (dict(num_k_heads=16, num_v_heads=40), "GDN_E_INVAL"),       # Hv not a multiple of Hk
    (dict(head_k_dim=96, head_v_dim=96), "GDN_E_UNSUPPORTED"),
    (dict(head_k_dim=128, head_v_dim=64), "GDN_E_UNSUPPORTED"),
    (dict(conv_width=3), "GDN_E_UNSUPPORTED"),
    (dict(l2_eps=-1.0), "GDN_E_INVAL"),
])
def test_bad_config_rejected(kw, status):
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_workspace_size(qwen_cfg(**kw), 4096, 1, 64)
    assert e.value.name == status


def test_workspace_size_and_bad_chunk():
    cfg = qwen_cfg()
    small = gdn.prefill_workspace_size(cfg, 4096, 1, 64)
    big = gdn.prefill_workspace_size(cfg, 65536, 16, 64)
    assert 0 < small < big
    # chunk 64 on bf16 d=128 holds the chunked form's intermediates: per token
    # q^, k^ (two fp16 parts) and v^, per (chunk, value head) a 65,664-byte record
    per_token = (2 * 2 * 16 * 128 + 48 * 128) * 2
    assert small >= 4096 * per_token + 64 * 48 * 65664
    # the affine chunked path runs chunks 16, 32 and 64 on bf16 d=128: per token q^, k^ (two parts) and,
    # per (64-row tile, value head), the two v^ images and the operand record
    for chunk in (16, 32):
        assert gdn.prefill_workspace_size(cfg, 4096, 1, chunk) >= 4096 * 2 * 2 * 16 * 128 * 2 + 64 * 48 * 32768
    f32 = gdn.make_config(gi.Geometry(io_dtype="f32"))
    sched_only = gdn.prefill_workspace_size(f32, 65536, 16, 16)  # token-recurrent path: the schedule alone
    assert 0 < sched_only < (1 << 20)
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_workspace_size(cfg, 4096, 1, 48)
    assert e.value.name == "GDN_E_INVAL"


def test_workspace_is_bounded_by_one_window():
    """The chunked paths run conv, prep and chain over windows of at most 65536 tokens, so beyond the
    schedule (16 bytes per chunk and a few per sequence) the workspace stops growing with the length."""
    cfg = qwen_cfg()
    for chunk in (16, 32, 64, 128):
        w1 = gdn.prefill_workspace_size(cfg, 65536, 1, chunk)
        w4 = gdn.prefill_workspace_size(cfg, 4 * 65536, 1, chunk)
        chunks = 3 * 65536 // min(chunk, 64)
        assert w1 < w4 <= w1 + 16 * chunks + 4096, (chunk, w1, w4)
        assert gdn.prefill_workspace_size(cfg, 4096, 1, chunk) < w1  # shorter inputs need less


class FakeTensor:
    """Host buffer with a data_ptr(), standing in for device memory in calls
    that must fail during validation (nothing may be written)."""

    def __init__(self, nbytes, fill=0x5A):
        self.buf = np.full(nbytes + 64, fill, np.uint8)
        off = (-self.buf.ctypes.data) % 64
        self.view = self.buf[off:off + nbytes]

    def data_ptr(self):
        return self.view.ctypes.data

    def numel(self):
        return self.view.size

    def element_size(self):
        return 1


def test_prefill_validation_rejects_before_launch():
    geo = gi.Geometry()
    cfg = gdn.make_config(geo)
    T = 8
    t = {k: FakeTensor(n) for k, n in dict(qkv=T * geo.conv_dim * 2, z=T * geo.value_dim * 2, a=T * 96, b=T * 96,
                                           o=T * geo.value_dim * 2, conv=3 * geo.conv_dim * 2,
                                           state=geo.num_v_heads * 128 * 128 * 4, ws=1 << 16).items()}
    params = tuple(FakeTensor(n) for n in (geo.conv_dim * 16, 192, 192, 512))
    cu_dev = FakeTensor(8)
    snapshot = {k: v.view.copy() for k, v in t.items()}

    def call(cu_host, chunk=64, flags=0, ws=t["ws"], wsb=None):
        gdn.prefill(cfg, params, t["qkv"], t["z"], t["a"], t["b"], cu_dev, cu_host, chunk, flags, t["conv"],
                    t["state"], t["o"], ws, workspace_bytes=wsb, stream=0)

    cases = [
        (dict(cu_host=[1, 8]), "GDN_E_INVAL"),            # cu[0] != 0
        (dict(cu_host=[0, 8, 4]), "GDN_E_INVAL"),         # decreasing
        (dict(cu_host=[0, 8], chunk=100), "GDN_E_INVAL"),
        (dict(cu_host=[0, 8], flags=0x80), "GDN_E_INVAL"),
        (dict(cu_host=[0, 8], flags=0x30), "GDN_E_INVAL"),   # two prefill paths at once
        (dict(cu_host=[0, 8], wsb=16), "GDN_E_WORKSPACE"),
    ]
    for kw, status in cases:
        with pytest.raises(gdn.GdnError) as e:
            call(**kw)
        assert e.value.name == status, (kw, e.value)
    # misaligned output pointer
    class Off(FakeTensor):
        def data_ptr(self):
            return self.view.ctypes.data + 2
    bad_o = Off(T * geo.value_dim * 2 + 16)
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill(cfg, params, t["qkv"], t["z"], t["a"], t["b"], cu_dev, [0, 8], 64, 0, t["conv"], t["state"],
                    bad_o, t["ws"], stream=0)
    assert e.value.name == "GDN_E_INVAL" and "aligned" in str(e.value)
    for k, v in t.items():
        assert np.array_equal(v.view, snapshot[k]), k


def test_prefill_noalloc_validates_cu_seqlens_host_on_the_host():
    """The no-scratch prefill names a NULL or malformed cu_seqlens_host itself,
    before it sizes anything from the array's last entry."""
    geo = gi.Geometry()
    cfg = gdn.make_config(geo)
    params = gdn._params(*(FakeTensor(n) for n in (geo.conv_dim * 16, 192, 192, 512)))
    t = FakeTensor(1 << 12)
    L = gdn.lib()

    def call(cu_ptr, n):
        return L.gdn_prefill_noalloc(ctypes.byref(cfg), ctypes.byref(params), t.data_ptr(), t.data_ptr(),
                                     t.data_ptr(), t.data_ptr(), t.data_ptr(), cu_ptr, n, 64, 0, t.data_ptr(),
                                     t.data_ptr(), t.data_ptr(), None)

    assert call(None, 1) == -1 and "cu_seqlens_host is NULL" in gdn.last_error()
    bad0 = np.array([4, 8], np.int32)
    assert call(bad0.ctypes.data, 1) == -1 and "cu_seqlens_host[0]" in gdn.last_error()
    dec = np.array([0, 8, 4], np.int32)
    assert call(dec.ctypes.data, 2) == -1 and "decreases" in gdn.last_error()


def test_prefill_noalloc_rejects_other_path_flags_on_the_host():
    """The no-scratch prefill runs the single-kernel path only: a flag that
    selects another path is named in the error, before any device call."""
    geo = gi.Geometry()
    cfg = gdn.make_config(geo)
    params = gdn._params(*(FakeTensor(n) for n in (geo.conv_dim * 16, 192, 192, 512)))
    t = FakeTensor(1 << 12)
    cu = np.array([0, 8], np.int32)
    L = gdn.lib()
    for f in (gdn.PREFILL_RECURRENT, gdn.PREFILL_FACTORED, gdn.PREFILL_AFFINE,
              gdn.PREFILL_AFFINE | gdn.ZERO_INIT_STATE):
        rc = L.gdn_prefill_noalloc(ctypes.byref(cfg), ctypes.byref(params), t.data_ptr(), t.data_ptr(),
                                   t.data_ptr(), t.data_ptr(), t.data_ptr(), cu.ctypes.data, 1, 64, f, t.data_ptr(),
                                   t.data_ptr(), t.data_ptr(), None)
        assert rc == -1 and "another prefill path" in gdn.last_error(), (f, gdn.last_error())


def test_decode_multi_validation_rejects_before_launch():
    """Draft counts outside 1..4, an accept array on a verify call and head
    dims other than 128 are refused on the host, with every buffer intact."""
    def bufs(geo, N, K):
        t = dict(qkv=FakeTensor(N * K * geo.conv_dim * 2), z=FakeTensor(N * K * geo.value_dim * 2),
                 a=FakeTensor(N * K * geo.num_v_heads * 2), b=FakeTensor(N * K * geo.num_v_heads * 2),
                 conv=FakeTensor(N * 3 * geo.conv_dim * 2), acc=FakeTensor(4 * N),
                 state=FakeTensor(N * geo.num_v_heads * geo.head_v_dim * geo.head_k_dim * 4),
                 o=FakeTensor(N * K * geo.value_dim * 2))
        params = tuple(FakeTensor(n) for n in (geo.conv_dim * 16, 4 * geo.num_v_heads, 4 * geo.num_v_heads,
                                               4 * geo.head_v_dim))
        return t, params

    geo = gi.Geometry(num_k_heads=2, num_v_heads=6)
    t, params = bufs(geo, 2, 2)
    snap = {k: v.view.copy() for k, v in t.items()}
    cfg = gdn.make_config(geo)
    for K, commit, acc, N, status in [(0, True, None, 2, "GDN_E_INVAL"), (5, True, None, 2, "GDN_E_INVAL"),
                                      (2, False, t["acc"], 2, "GDN_E_INVAL"), (2, True, None, 0, "GDN_E_INVAL")]:
        with pytest.raises(gdn.GdnError) as e:
            gdn.decode_multi(cfg, params, t["qkv"], t["z"], t["a"], t["b"], N, K, commit, acc, t["conv"],
                             t["state"], t["o"], stream=0)
        assert e.value.name == status, (K, commit, N)
    geo64 = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=64, head_v_dim=64)
    t64, params64 = bufs(geo64, 2, 2)
    with pytest.raises(gdn.GdnError) as e:
        gdn.decode_multi(gdn.make_config(geo64), params64, t64["qkv"], t64["z"], t64["a"], t64["b"], 2, 2, True,
                         None, t64["conv"], t64["state"], t64["o"], stream=0)
    assert e.value.name == "GDN_E_UNSUPPORTED"
    for k, v in t.items():
        assert np.array_equal(v.view, snap[k]), k


# ---------------------------------------------------------------- state blobs (host memory)

MAGIC = b"GDNSTATE"


def mix64(z):
    M = (1 << 64) - 1
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
    return z ^ (z >> 31)


def checksum(payload: bytes) -> int:
    w = np.frombuffer(payload, dtype="<u8")
    M = (1 << 64) - 1
    s = 0
    for i, x in enumerate(w.tolist()):
        s = (s + mix64((x + (i + 1) * 0x9E3779B97F4A7C15) & M)) & M
    return s


def make_blob(geo, version=1, io_dtype=None, layout=1, corrupt_payload=False, hk=None):
    cb = 3 * geo.conv_dim * geo.io_bytes
    sb = geo.num_v_heads * geo.head_v_dim * geo.head_k_dim * 4
    rng = np.random.default_rng(0)
    payload = rng.integers(0, 256, cb + sb, dtype=np.uint8).tobytes()
    io = (1 if geo.io_dtype == "bf16" else 0) if io_dtype is None else io_dtype
    hdr = struct.pack("<8sII8iQQQ", MAGIC, version, 128, hk or geo.num_k_heads, geo.num_v_heads, geo.head_k_dim,
                      geo.head_v_dim, geo.conv_width, io, 0, layout, cb, sb, checksum(payload))
    hdr = hdr + bytes(128 - len(hdr))
    if corrupt_payload:
        payload = payload[:100] + bytes([payload[100] ^ 1]) + payload[101:]
    return np.frombuffer(hdr + payload, np.uint8).copy()


def test_blob_size_matches_layout():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32)
    assert gdn.state_blob_size(gdn.make_config(geo)) == 128 + 3 * geo.conv_dim * 2 + 4 * 32 * 32 * 4


@pytest.mark.parametrize("mut,status", [
    (lambda b: b.__setitem__(0, ord("X")), "GDN_E_BLOB_FORMAT"),
    (None, "GDN_E_BLOB_VERSION"),
    (None, "GDN_E_BLOB_GEOMETRY"),
    (None, "GDN_E_BLOB_CHECKSUM"),
    (None, "GDN_E_BLOB_FORMAT_LAYOUT"),
    (None, "GDN_E_BLOB_GEOMETRY_DTYPE"),
])
def test_corrupt_host_blob_rejected_without_writes(mut, status):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32)
    cfg = gdn.make_config(geo)
    if status == "GDN_E_BLOB_VERSION":
        blob = make_blob(geo, version=2)
    elif status == "GDN_E_BLOB_GEOMETRY":
        blob = make_blob(geo, hk=1)
    elif status == "GDN_E_BLOB_CHECKSUM":
        blob = make_blob(geo, corrupt_payload=True)
    elif status == "GDN_E_BLOB_FORMAT_LAYOUT":
        blob, status = make_blob(geo, layout=7), "GDN_E_BLOB_FORMAT"
    elif status == "GDN_E_BLOB_GEOMETRY_DTYPE":
        blob, status = make_blob(geo, io_dtype=0), "GDN_E_BLOB_GEOMETRY"
    else:
        blob = make_blob(geo)
        mut(blob)
    conv = FakeTensor(3 * geo.conv_dim * 2)
    st = FakeTensor(4 * 32 * 32 * 4)
    c0, s0 = conv.view.copy(), st.view.copy()
    with pytest.raises(gdn.GdnError) as e:
        gdn.state_restore(cfg, blob, 0, conv, st, stream=0)
    assert e.value.name == status, e.value
    assert np.array_equal(conv.view, c0) and np.array_equal(st.view, s0)


def test_truncated_blob_rejected():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32)
    blob = make_blob(geo)[:-8]
    with pytest.raises(gdn.GdnError) as e:
        gdn.state_restore(gdn.make_config(geo), blob, 0, FakeTensor(4096), FakeTensor(65536), stream=0)
    assert e.value.name == "GDN_E_BLOB_FORMAT"


def test_projection_validation_rejects_before_launch():
    """Bad K (not a positive multiple of 8), a bad tile width, a NULL or odd
    output and a non-bf16 config are refused on the host, buffers intact."""
    L = gdn.lib()
    x, w, y = FakeTensor(64 * 64 * 2), FakeTensor(64 * 64 * 2), FakeTensor(64 * 64 * 2)
    snap = {k: t.view.copy() for k, t in dict(x=x, w=w, y=y).items()}
    cases = [
        (dict(M=4, K=12, N=8, y=y.data_ptr(), tile_n=0), "GDN_E_INVAL"),
        (dict(M=4, K=0, N=8, y=y.data_ptr(), tile_n=0), "GDN_E_INVAL"),
        (dict(M=-1, K=16, N=8, y=y.data_ptr(), tile_n=0), "GDN_E_INVAL"),
        (dict(M=4, K=16, N=8, y=y.data_ptr(), tile_n=80), "GDN_E_INVAL"),
        (dict(M=4, K=16, N=8, y=y.data_ptr(), tile_n=288), "GDN_E_INVAL"),
        (dict(M=4, K=16, N=8, y=None, tile_n=0), "GDN_E_INVAL"),
        (dict(M=4, K=16, N=8, y=y.data_ptr() + 1, tile_n=0), "GDN_E_INVAL"),
    ]
    for c, status in cases:
        rc = L.gdn_gemm_bf16(x.data_ptr(), c["M"], c["K"], w.data_ptr(), c["N"], c["y"], c["tile_n"], None)
        assert gdn.STATUS[rc] == status, (c, gdn.last_error())
    rc = L.gdn_gemm_bf16(x.data_ptr() + 2, 4, 16, w.data_ptr(), 8, y.data_ptr(), 0, None)
    assert gdn.STATUS[rc] == "GDN_E_INVAL" and "aligned" in gdn.last_error()
    geo32 = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32, io_dtype="f32")
    with pytest.raises(gdn.GdnError) as e:
        L2 = np.zeros((4, 64), np.uint16)
        gdn.project_in(gdn.make_config(geo32), L2, np.zeros((8, 64), np.uint16), y, y, y, y, stream=0)
    assert e.value.name == "GDN_E_UNSUPPORTED"
    with pytest.raises(gdn.GdnError) as e:
        gdn.project_out(gdn.make_config(geo32), np.zeros((4, 128), np.uint16), np.zeros((8, 128), np.uint16), y,
                        stream=0)
    assert e.value.name == "GDN_E_UNSUPPORTED"
    for k, t in dict(x=x, w=w, y=y).items():
        assert np.array_equal(t.view, snap[k]), k


def test_seqpar_validation_and_workspace():
    """gdn_prefill_seqpar takes bf16 with d = 128 only; bad segment counts and
    flags are refused on the host, buffers intact; the workspace grows with
    the segment count (3 fp32 states per segment and value head)."""
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6)
    cfg = gdn.make_config(geo)
    w4 = gdn.prefill_seqpar_workspace_size(cfg, 65536, 4)
    w8 = gdn.prefill_seqpar_workspace_size(cfg, 65536, 8)
    assert w8 - w4 >= 3 * 4 * geo.num_v_heads * 128 * 128 * 4
    # the factored chunked form's intermediates (q^, k^ in two parts; a 123,520-byte record per (chunk,
    # value head)) plus the segment states
    assert w4 > 65536 * 2 * 2 * geo.num_k_heads * 128 * 2 + 1024 * geo.num_v_heads * 123520
    for g, status in [(gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=64, head_v_dim=64), "GDN_E_UNSUPPORTED"),
                      (gi.Geometry(num_k_heads=2, num_v_heads=6, io_dtype="f32"), "GDN_E_UNSUPPORTED")]:
        with pytest.raises(gdn.GdnError) as e:
            gdn.prefill_seqpar_workspace_size(gdn.make_config(g), 1000, 0)
        assert e.value.name == status
    for T, seg in [(-1, 0), (1000, -2), (1000, 5000)]:
        with pytest.raises(gdn.GdnError) as e:
            gdn.prefill_seqpar_workspace_size(cfg, T, seg)
        assert e.value.name == "GDN_E_INVAL"
    t = dict(qkv=FakeTensor(100 * geo.conv_dim * 2), z=FakeTensor(100 * geo.value_dim * 2),
             a=FakeTensor(100 * 6 * 2), b=FakeTensor(100 * 6 * 2), conv=FakeTensor(3 * geo.conv_dim * 2),
             state=FakeTensor(6 * 128 * 128 * 4), o=FakeTensor(100 * geo.value_dim * 2), ws=FakeTensor(w4))
    params = tuple(FakeTensor(n) for n in (geo.conv_dim * 16, 24, 24, 512))
    snap = {k: v.view.copy() for k, v in t.items()}
    cases = [(gdn.PREFILL_RECURRENT, t["ws"], "GDN_E_INVAL"),   # only the two ZERO_INIT flags
             (0, None, "GDN_E_WORKSPACE")]
    for flags, ws, status in cases:
        with pytest.raises(gdn.GdnError) as e:
            gdn.prefill_seqpar(cfg, params, t["qkv"], t["z"], t["a"], t["b"], 100, 2, flags, t["conv"], t["state"],
                               t["o"], ws, workspace_bytes=0 if ws is None else None, stream=0)
        assert e.value.name == status
    for k, v in t.items():
        assert np.array_equal(v.view, snap[k]), k


def test_header_is_plain_c(tmp_path):
    """include/gdn.h compiles as C99 and a C program links against libgdn.so
    and calls entry points that need no GPU."""
    import subprocess
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "gdn.h"\n#include <stdio.h>\n#include <string.h>\n'
        'int main(void) {\n'
        '  gdn_config cfg; size_t bytes = 0; memset(&cfg, 0, sizeof cfg);\n'
        '  cfg.num_k_heads = 16; cfg.num_v_heads = 48; cfg.head_k_dim = 128; cfg.head_v_dim = 128;\n'
        '  cfg.conv_width = 4; cfg.l2_eps = 1e-6f; cfg.norm_eps = 1e-6f; cfg.q_scale = 1.0f; cfg.io_dtype = GDN_BF16;\n'
        '  if (gdn_prefill_workspace_size(&cfg, 4096, 1, 64, &bytes) != GDN_OK || bytes == 0) return 2;\n'
        '  if (gdn_gemm_bf16(NULL, 4, 12, NULL, 8, NULL, 0, NULL) != GDN_E_INVAL) return 3;\n'
        '  printf("%d %s %zu\\n", gdn_abi_version(), gdn_kernel_name(GDN_K_DECODE), bytes);\n'
        '  return 0;\n}\n')
    lib_dir = os.path.join(ROOT, "linear_attention_recurrence_deltanet_b200")
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", lib_dir, "-lgdn", "-Wl,-rpath," + lib_dir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[0] == "1" and out[1] == "decode" and int(out[2]) > 0
