"""The C-ABI library loads without a GPU, exports every symbol include/sas.h
declares, and rejects bad arguments on the host before any launch.

No test here launches a kernel: every call below fails validation first, so
it runs on a machine without a GPU driver.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sas.h")


@pytest.fixture(scope="module")
def raw():
    from block_sparse_attention_sas_b200 import build as B
    B.build()
    from block_sparse_attention_sas_b200 import _lib
    return _lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sas_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(raw):
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(raw.LIB, n), n
    assert set(names) == set(raw.SIGNATURES), "binding and header disagree"


def test_status_strings_and_version(raw):
    for code, name in raw.STATUS.items():
        assert raw.LIB.sas_status_string(code).decode() == name
    assert raw.LIB.sas_status_string(99).decode() == "SAS_ERR_UNKNOWN"
    assert raw.LIB.sas_version() == 100


FAKE = ctypes.c_void_p(1 << 20)        # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


def fwd(raw, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, v=FAKE, idx=FAKE, gates=None, B=1, Hq=4, Hkv=2, T=128, d=128,
             b=64, K=2, scale=0.0, o=FAKE, lse=FAKE)
    a.update(kw)
    return raw.LIB.sas_attn_fwd(a["dtype"], a["q"], a["k"], a["v"], a["idx"], a["gates"], a["B"],
                                a["Hq"], a["Hkv"], a["T"], a["d"], a["b"], a["K"], a["scale"],
                                a["o"], a["lse"], None)


@pytest.mark.parametrize("kw,want", [
    (dict(dtype=7), 1), (dict(q=None), 1), (dict(o=None), 1), (dict(idx=None), 1),
    (dict(Hq=3), 1), (dict(K=0), 1), (dict(T=0), 1), (dict(scale=float("nan")), 1),
    (dict(q=MISALIGNED), 1), (dict(d=96), 2), (dict(b=128), 2), (dict(K=300), 2),
])
def test_fwd_rejects(raw, kw, want):
    assert fwd(raw, **kw) == want


def test_empty_batch_is_a_no_op(raw):
    assert fwd(raw, B=0, q=None, k=None, v=None, o=None, lse=None, idx=None) == 0
    assert raw.LIB.sas_gate_topk(None, 0, 8, 16, 16, 1, 4, None, None, None) == 0


def test_gate_topk_rejects(raw):
    L = raw.LIB
    assert L.sas_gate_topk(FAKE, 1, 1, 16, 16, 2, 4, FAKE, FAKE, None) == 1   # causal flag
    assert L.sas_gate_topk(FAKE, 1, 1, 8, 16, 1, 4, FAKE, FAKE, None) == 1    # causal rows != C
    assert L.sas_gate_topk(FAKE, 1, 1, 1, 16, 0, 0, FAKE, FAKE, None) == 1    # K = 0
    assert L.sas_gate_topk(FAKE, 1, 1, 1, 16, 0, 300, FAKE, FAKE, None) == 2  # K too large
    assert L.sas_gate_topk(None, 1, 1, 1, 16, 0, 4, FAKE, FAKE, None) == 1
    assert L.sas_gate_topk(FAKE, 1, 1, 1, 1 << 20, 0, 4, FAKE, FAKE, None) == 2


def test_bwd_workspace_and_gate_rules(raw):
    L = raw.LIB
    need = L.sas_attn_bwd_workspace_size(1, 1, 32, 8, 16384, 128, 64, 16)
    assert need > 4 * 32 * 16384  # at least the per-row D vector
    # bf16 with the tensor-core shape also holds the dS tiles: 8*256*2*17 of 16 KB
    assert need > 8 * 256 * 2 * 17 * 16384
    assert L.sas_attn_bwd_workspace_size(0, 1, 32, 8, 16384, 128, 64, 16) < need  # fp32: no tiles
    assert L.sas_attn_bwd_workspace_size(1, 1, 3, 2, 128, 128, 64, 2) == 0  # invalid shape

    def bwd(ws, ws_bytes, gates=None, ds=None):
        return L.sas_attn_bwd(1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, gates, 1, 32, 8, 16384,
                              128, 64, 16, 0.0, FAKE, FAKE, FAKE, ds, ws, ws_bytes, None)
    assert bwd(FAKE, need - 1) == 5
    assert bwd(None, need) == 5
    assert bwd(MISALIGNED, need) == 5
    assert bwd(FAKE, need, gates=None, ds=FAKE) == 1  # dscores needs gates


def test_decode_rejects(raw):
    L = raw.LIB
    need = L.sas_decode_workspace_size(8, 32, 8, 65536, 128, 64, 32)
    assert need > 0

    def dec(**kw):
        a = dict(dtype=1, q=FAKE, kc=FAKE, vc=FAKE, idx=FAKE, gates=None, use=0, B=8, Hq=32, Hkv=8,
                 L=65536, Lcap=65536, d=128, b=64, K=32, o=FAKE, ws=FAKE, wsb=need)
        a.update(kw)
        return L.sas_decode(a["dtype"], a["q"], a["kc"], a["vc"], a["idx"], a["gates"], a["use"],
                            a["B"], a["Hq"], a["Hkv"], a["L"], a["Lcap"], a["d"], a["b"], a["K"],
                            0.0, a["o"], a["ws"], a["wsb"], None)
    assert dec(use=1, gates=None) == 1      # gates required when use_gates
    assert dec(L=70000) == 1                # L > Lcap
    assert dec(Hq=72, Hkv=8) == 2           # G = 9 > 8
    assert dec(wsb=need - 1) == 5
    assert dec(kc=MISALIGNED) == 1


def test_wait_limit_setter_is_host_only(raw):
    raw.LIB.sas_set_wait_limit(1000)
    raw.LIB.sas_set_wait_limit(0)


def test_gate_variant_arguments_are_checked(raw):
    """Unknown gate activations or gatings are rejected before any launch."""
    L = raw.LIB
    st = L.sas_gate_topk_phi(FAKE, 1, 1, 4, 4, 1, 2, 3, FAKE, FAKE, None)
    assert st == 1
    a = (1, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, 128, 64, 2, 0.0)
    assert L.sas_attn_fwd_gated(*a, 2, FAKE, FAKE, None) == 1
    assert L.sas_attn_fwd_gated(*a, -1, FAKE, FAKE, None) == 1
    b = (1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, 128, 64, 2, 0.0)
    assert L.sas_attn_bwd_gated(*b, 5, 0, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None) == 1
    assert L.sas_attn_bwd_gated(*b, 0, 9, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None) == 1
