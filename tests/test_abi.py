"""The C ABI boundary without a GPU: the library loads, exports every symbol that
include/gdr.h declares, and rejects bad arguments with the documented status codes
before anything is launched (the calls below never reach a launch: each carries at
least one error that the checks catch first)."""

import ctypes
import os
import re

import pytest

import gated_delta_rule_145_b200 as gdr

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "gdr.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDR_API\s+[\w\s\*]*?\b(gdr_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("gdr_prefill_chunked", "gdr_decode_step", "gdr_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(gdr.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, f"not exported: {missing}"


def test_status_strings():
    for code in (gdr.GDR_OK, gdr.GDR_ERR_NULL, gdr.GDR_ERR_SHAPE, gdr.GDR_ERR_UNSUPPORTED,
                 gdr.GDR_ERR_ALIGN, gdr.GDR_ERR_CUDA):
        assert gdr.gdr_status_string(code).startswith("GDR_")


# fake, 256-byte aligned addresses: never dereferenced, because every case below fails a
# host-side check first
A = 1 << 20


def _prefill(name="gdr_prefill_chunked", **kw):
    args = dict(q=A, k=A + 256, v=A + 512, a=A + 768, b=A + 1024, A_log=A + 1280,
                dt_bias=A + 1536, init_state=None, out=A + 2048, final_state=None,
                cu_seqlens=None, B=1, T=64, Hk=4, Hv=4, dk=128, dv=128, chunk=32)
    args.update(kw)
    fn = getattr(gdr, name)
    if name.startswith("gdr_prefill_recurrent"):
        args.pop("chunk")
    return fn(**args, stream=0, check=False)


@pytest.mark.parametrize("name", ["gdr_prefill_chunked", "gdr_prefill_chunked_f32",
                                  "gdr_prefill_recurrent", "gdr_prefill_recurrent_f32"])
def test_prefill_argument_errors(name):
    assert _prefill(name, q=None) == gdr.GDR_ERR_NULL
    assert _prefill(name, out=None) == gdr.GDR_ERR_NULL
    assert _prefill(name, A_log=None) == gdr.GDR_ERR_NULL
    assert _prefill(name, Hk=3, Hv=4) == gdr.GDR_ERR_SHAPE
    assert _prefill(name, B=0) == gdr.GDR_ERR_SHAPE
    assert _prefill(name, T=-1) == gdr.GDR_ERR_SHAPE
    assert _prefill(name, Hk=0) == gdr.GDR_ERR_SHAPE
    assert _prefill(name, dk=96, dv=96) == gdr.GDR_ERR_UNSUPPORTED
    assert _prefill(name, dk=128, dv=64) == gdr.GDR_ERR_UNSUPPORTED
    assert _prefill(name, q=A + 8) == gdr.GDR_ERR_ALIGN
    assert _prefill(name, out=A + 2052) == gdr.GDR_ERR_ALIGN
    assert _prefill(name, init_state=A + 4) == gdr.GDR_ERR_ALIGN
    if "chunked" in name:
        assert _prefill(name, chunk=16) == gdr.GDR_ERR_UNSUPPORTED
        assert _prefill(name, chunk=64) == gdr.GDR_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["gdr_decode_step", "gdr_decode_step_f32"])
def test_decode_argument_errors(name):
    fn = getattr(gdr, name)

    def call(**kw):
        args = dict(q=A, k=A + 256, v=A + 512, a=A + 768, b=A + 1024, A_log=A + 1280,
                    dt_bias=A + 1536, state=A + 4096, out=A + 2048, B=2, Hk=4, Hv=8, dk=128,
                    dv=128)
        args.update(kw)
        return fn(**args, stream=0, check=False)

    assert call(state=None) == gdr.GDR_ERR_NULL
    assert call(v=None) == gdr.GDR_ERR_NULL
    assert call(Hv=6) == gdr.GDR_ERR_SHAPE
    assert call(B=0) == gdr.GDR_ERR_SHAPE
    assert call(dk=48, dv=48) == gdr.GDR_ERR_UNSUPPORTED
    assert call(state=A + 4100) == gdr.GDR_ERR_ALIGN


def test_binding_rejects_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 4, 1, 32)
    with pytest.raises(ValueError, match="CUDA"):
        gdr.prefill(x, x, x, torch.zeros(1, 4, 1), torch.zeros(1, 4, 1), torch.zeros(1),
                    torch.zeros(1))


def test_mixer_io_argument_errors():
    conv = lambda **kw: gdr.gdr_short_conv_silu(**{**dict(
        x=A, weight=A + 256, bias=None, conv_state_in=None, conv_state_out=None, y=A + 512,
        B=1, T=16, C=64, width=4), **kw}, stream=0, check=False)
    assert conv(x=None) == gdr.GDR_ERR_NULL
    assert conv(C=60) == gdr.GDR_ERR_SHAPE
    assert conv(B=0) == gdr.GDR_ERR_SHAPE
    assert conv(width=3) == gdr.GDR_ERR_UNSUPPORTED
    assert conv(y=A + 8) == gdr.GDR_ERR_ALIGN
    norm = lambda fn=gdr.gdr_gated_rmsnorm, **kw: fn(**{**dict(
        o=A, z=A + 256, weight=A + 512, y=A + 768, rows=10, d=128, eps=1e-6), **kw},
        stream=0, check=False)
    assert norm(o=None) == gdr.GDR_ERR_NULL
    assert norm(d=96) == gdr.GDR_ERR_UNSUPPORTED
    assert norm(rows=-1) == gdr.GDR_ERR_SHAPE
    assert norm(eps=-1.0) == gdr.GDR_ERR_SHAPE
    assert norm(y=A + 8) == gdr.GDR_ERR_ALIGN
    assert norm(gdr.gdr_gated_rmsnorm_f32, z=A + 8) == gdr.GDR_ERR_ALIGN
