"""The C ABI: library loads, exports every declared symbol, rejects bad
arguments synchronously (no device needed for any of these)."""
import ctypes
import os
import re

import pytest

from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return binding.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(binding.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code, name in enumerate(["KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                 "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT", "KDA_ERR_INPUT_RANGE"]):
        assert binding.status_string(code) == name


def test_workspace_bytes(lib):
    f = lib.kda_chunk_prefill_workspace_bytes
    assert f(1000, 1, 4, 64, 64, binding.KDA_F32) == 0          # fp32 path: no workspace
    assert f(1000, 1, 4, 96, 96, binding.KDA_BF16) == 0         # unsupported size
    w1 = f(64 * 10, 1, 4, 128, 128, binding.KDA_BF16)
    w2 = f(64 * 10, 3, 4, 128, 128, binding.KDA_BF16)
    assert w1 > 0 and w2 > w1                                    # bound grows with N
    assert w1 % 256 == 0
    # upper bound holds for any split of the rows into N sequences
    assert f(0, 0, 1, 128, 128, binding.KDA_BF16) >= 0


def _args(**kw):
    base = dict(q=1, k=2, v=3, g=4, beta=5, o=6, B=1, T=16, N=1, H=2, dk=64, dv=64,
                dtype=binding.KDA_F32)
    base.update(kw)
    return base


@pytest.mark.parametrize("bad", [
    dict(B=-1), dict(T=-5), dict(H=0), dict(N=2),                   # N must equal B
    dict(q=None), dict(o=None), dict(dtype=7),
    dict(cu_seqlens=9, B=2),                                         # packed needs B == 1
])
def test_prefill_rejects_invalid_arguments(lib, bad):
    assert binding.raw_prefill(_args(**bad)) == binding.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(dk=96, dv=96), dict(dk=64, dv=128), dict(dk=32, dv=32)])
def test_prefill_rejects_unsupported_sizes(lib, bad):
    assert binding.raw_prefill(_args(**bad)) == binding.KDA_ERR_UNSUPPORTED


def test_prefill_bf16_requires_workspace(lib):
    a = _args(dtype=binding.KDA_BF16, dk=128, dv=128)
    assert binding.raw_prefill(a) == binding.KDA_ERR_INVALID_ARG
    need = lib.kda_chunk_prefill_workspace_bytes(16, 1, 2, 128, 128, binding.KDA_BF16)
    a.update(workspace=4096, workspace_bytes=need - 1)
    assert binding.raw_prefill(a) == binding.KDA_ERR_INVALID_ARG
    a.update(workspace=4096 + 16, workspace_bytes=need)           # not 256-byte aligned
    assert binding.raw_prefill(a) == binding.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("which", ["q", "k", "v", "g"])
def test_prefill_bf16_requires_16_byte_aligned_tiles(lib, which):
    """The tensor-core path loads q, k, g and v as TMA tiles: a base that is not
    16-byte aligned is refused before anything is launched."""
    need = lib.kda_chunk_prefill_workspace_bytes(16, 1, 2, 128, 128, binding.KDA_BF16)
    a = _args(dtype=binding.KDA_BF16, dk=128, dv=128, q=1 << 20, k=2 << 20, v=3 << 20,
              g=4 << 20, beta=5 << 20, o=6 << 20, workspace=8 << 20, workspace_bytes=need)
    a[which] += 8
    assert binding.raw_prefill(a) == binding.KDA_ERR_INVALID_ARG


def test_prefill_zero_sequences_is_a_no_op(lib):
    # N = B = 0: nothing to do, nothing launched
    assert binding.raw_prefill(_args(B=0, N=0, q=None, k=None, v=None, g=None, beta=None,
                                     o=None)) == binding.KDA_OK


def _dargs(**kw):
    base = dict(q=1, k=2, v=3, g=4, beta=5, state=16, o=6, N=4, H=2, dk=128, dv=128,
                dtype=binding.KDA_BF16)
    base.update(kw)
    return base


@pytest.mark.parametrize("bad", [dict(N=-1), dict(H=0), dict(state=None), dict(o=None),
                                 dict(dtype=3), dict(state=18)])   # state must be 16B aligned
def test_decode_rejects_invalid_arguments(lib, bad):
    assert binding.raw_decode(_dargs(**bad)) == binding.KDA_ERR_INVALID_ARG


def test_decode_rejects_unsupported_sizes(lib):
    assert binding.raw_decode(_dargs(dk=128, dv=64)) == binding.KDA_ERR_UNSUPPORTED


def test_decode_zero_sequences_is_a_no_op(lib):
    assert binding.raw_decode(_dargs(N=0)) == binding.KDA_OK


# ---------------------------------------------------------------- intermediate states

def test_checkpoint_count_dense_and_packed(lib):
    count = lambda cu, B, T, N, iv: lib.kda_prefill_checkpoint_count(cu, B, T, N, iv)
    assert count(None, 3, 1000, 3, 128) == 3 * 7          # 128 .. 896 inside 1000 tokens
    assert count(None, 2, 1024, 2, 512) == 2 * 1          # 512 only; 1024 is state_out
    assert count(None, 1, 0, 1, 64) == 0
    cu = (ctypes.c_int32 * 5)(0, 64, 64, 700, 1000)     # lengths 64, 0, 636, 300
    assert count(cu, 1, 1000, 4, 64) == 0 + 0 + 9 + 4
    bad = (ctypes.c_int32 * 4)(0, 900, 500, 5000)        # clamped to 0, 900, 900, 1000
    assert count(bad, 1, 1000, 3, 256) == 3 + 0 + 0
    assert count(None, 2, 10, 2, 0) == -1 and count(None, 2, 10, 3, 64) == -1


def _cargs(**kw):
    base = _args(interval=128, ckpt=64, ckpt_capacity=4, dtype=binding.KDA_BF16, dk=128, dv=128)
    base.update(kw)
    return base


@pytest.mark.parametrize("bad,code", [
    (dict(interval=0), "KDA_ERR_INVALID_ARG"), (dict(interval=-64), "KDA_ERR_INVALID_ARG"),
    (dict(ckpt=None), "KDA_ERR_INVALID_ARG"), (dict(ckpt=72), "KDA_ERR_INVALID_ARG"),
    (dict(ckpt_capacity=-1), "KDA_ERR_INVALID_ARG"),
    (dict(interval=100), "KDA_ERR_UNSUPPORTED"), (dict(dtype=binding.KDA_F32), "KDA_ERR_UNSUPPORTED")])
def test_checkpointed_prefill_rejects(lib, bad, code):
    assert binding.raw_prefill_checkpointed(_cargs(**bad)) == getattr(binding, code)


def _xargs(**kw):
    base = dict(_args(dtype=binding.KDA_BF16), flags=0, ckpt_interval=0, ckpt=None,
                ckpt_capacity=0)
    base.update(kw)
    return base


def raw_ex(a):
    return int(binding.load().kda_chunk_prefill_ex(
        a.get("q"), a.get("k"), a.get("v"), a.get("g"), a.get("beta"), a.get("state_in"),
        a.get("cu_seqlens"), a["B"], a["T"], a["N"], a["H"], a["dk"], a["dv"], a["dtype"],
        a["flags"], a.get("o"), a.get("state_out"), a["ckpt_interval"], a.get("ckpt"),
        a["ckpt_capacity"], a.get("workspace"), a.get("workspace_bytes", 0), a.get("stream")))


@pytest.mark.parametrize("bad,code", [
    (dict(flags=4), "KDA_ERR_INVALID_ARG"), (dict(ckpt_interval=-64), "KDA_ERR_INVALID_ARG"),
    (dict(ckpt_capacity=2), "KDA_ERR_INVALID_ARG"),                       # capacity without array
    (dict(flags=1, dtype=binding.KDA_F32), "KDA_ERR_UNSUPPORTED"),
    (dict(ckpt_interval=100, ckpt=64, ckpt_capacity=1), "KDA_ERR_UNSUPPORTED"),
    (dict(flags=3), "KDA_ERR_UNSUPPORTED"),      # preprocessing needs the d = 128 bf16 path
    (dict(flags=3, dk=128, dv=128), "KDA_ERR_INVALID_ARG")])   # no workspace given
def test_prefill_ex_rejects(lib, bad, code):
    assert raw_ex(_xargs(**bad)) == getattr(binding, code)


def test_backward_workspace_bytes(lib):
    states = ((1000 + 63) // 64 + 1) * 2 * 128 * 128 * 4 + 1 * 2 * 64 * 128 * 128 * 4
    # 2 units: four value-column slices, each with its partial sums of dq, dk, da, dbeta
    partials = 4 * 1000 * 2 * (3 * 128 + 4) * 4
    assert lib.kda_backward_workspace_bytes(1000, 1, 2, 128, 128) == states + partials
    # 50 units: two slices; 100 units: one, no partials
    assert lib.kda_backward_workspace_bytes(1000, 1, 50, 64, 64) == \
        ((1000 + 63) // 64 + 1) * 50 * 64 * 64 * 4 + 50 * 64 * 64 * 64 * 4 + 2 * 1000 * 50 * (3 * 64 + 4) * 4
    assert lib.kda_backward_workspace_bytes(1000, 1, 100, 64, 64) == \
        ((1000 + 63) // 64 + 1) * 100 * 64 * 64 * 4 + 100 * 64 * 64 * 64 * 4
    assert lib.kda_backward_workspace_bytes(10, 1, 2, 96, 96) == 0


def _bargs(**kw):
    base = dict(q=16, k=32, v=48, g=64, beta=80, state_in=None, cu=None, B=1, T=16, N=1, H=2,
                dk=64, dv=64, dtype=binding.KDA_F32, do=96, ds=None, dq=112, dkk=128, dvv=144,
                dg=160, db=176, ds0=None, ws=None, wsb=0)
    base.update(kw)
    return base


def raw_bwd(a):
    return int(binding.load().kda_backward(
        a["q"], a["k"], a["v"], a["g"], a["beta"], a["state_in"], a["cu"], a["B"], a["T"], a["N"],
        a["H"], a["dk"], a["dv"], a["dtype"], a["do"], a["ds"], a["dq"], a["dkk"], a["dvv"],
        a["dg"], a["db"], a["ds0"], a["ws"], a["wsb"], None))


@pytest.mark.parametrize("bad,code", [
    (dict(B=-1), "KDA_ERR_INVALID_ARG"), (dict(N=2), "KDA_ERR_INVALID_ARG"),
    (dict(do=None), "KDA_ERR_INVALID_ARG"), (dict(dg=None), "KDA_ERR_INVALID_ARG"),
    (dict(dtype=5), "KDA_ERR_INVALID_ARG"), (dict(state_in=8), "KDA_ERR_INVALID_ARG"),
    (dict(dk=96, dv=96), "KDA_ERR_UNSUPPORTED"),
    (dict(), "KDA_ERR_INVALID_ARG"),             # no workspace
    # the chunked form (bf16, d = 128) reads do and writes dv in 16-byte pieces
    (dict(dtype=binding.KDA_BF16, dk=128, dv=128, ws=256, wsb=1 << 40, do=104),
     "KDA_ERR_INVALID_ARG"),
    (dict(dtype=binding.KDA_BF16, dk=128, dv=128, ws=256, wsb=1 << 40, dvv=136),
     "KDA_ERR_INVALID_ARG")])
def test_backward_rejects(lib, bad, code):
    assert raw_bwd(_bargs(**bad)) == getattr(binding, code)


def test_backward_zero_sequences_is_a_no_op(lib):
    assert raw_bwd(_bargs(B=0, N=0)) == binding.KDA_OK


def _iargs(**kw):
    base = _dargs(slots=64, P=4)
    base.update(kw)
    return base


@pytest.mark.parametrize("bad", [dict(N=-1), dict(P=-1), dict(H=0), dict(state=None),
                                 dict(slots=None), dict(o=None), dict(dtype=3), dict(state=18)])
def test_decode_indexed_rejects_invalid_arguments(lib, bad):
    assert binding.raw_decode_indexed(_iargs(**bad)) == binding.KDA_ERR_INVALID_ARG


def test_decode_indexed_rejects_unsupported_sizes(lib):
    assert binding.raw_decode_indexed(_iargs(dk=128, dv=64)) == binding.KDA_ERR_UNSUPPORTED


def test_decode_indexed_zero_requests_is_a_no_op(lib):
    assert binding.raw_decode_indexed(_iargs(N=0)) == binding.KDA_OK


def test_selftest_rejects_bad_limits(lib):
    assert lib.kda_selftest_bounded_wait(0, None) == binding.KDA_ERR_INVALID_ARG
    assert lib.kda_selftest_bounded_wait(10**7 + 1, None) == binding.KDA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="libkda.so not found"):
        binding.load(str(tmp_path / "nope.so"))


def test_host_prefill_workspace_bytes(lib):
    al = lambda x: (x + 255) // 256 * 256
    H, d = 2, 128
    # T = 1000 < the default segment: one segment of 1024 rows (T rounded up to the chunk)
    rows = 1024
    pre = al(lib.kda_chunk_prefill_workspace_bytes(rows, 1, H, d, d, binding.KDA_BF16))
    ins = 4 * al(rows * H * d * 2) + al(rows * H * 2)
    want = 2 * ins + 2 * al(rows * H * d * 4) + 2 * al(H * d * d * 4) + pre
    assert lib.kda_prefill_host_workspace_bytes(1, 1000, H, d, d, binding.KDA_BF16, 0) == want
    # an explicit segment sizes the buffers, whatever T is
    rows = 3 * 256
    pre = al(lib.kda_chunk_prefill_workspace_bytes(rows, 3, H, 64, 64, binding.KDA_F32))
    ins = 4 * al(rows * H * 64 * 4) + al(rows * H * 4)
    want = 2 * ins + 2 * al(rows * H * 64 * 4) + 2 * al(3 * H * 64 * 64 * 4) + pre
    assert lib.kda_prefill_host_workspace_bytes(3, 5000, H, 64, 64, binding.KDA_F32, 256) == want
    for bad in ((1, 1000, H, d, d, binding.KDA_BF16, 100),    # segment not a multiple of 64
                (1, 1000, H, 96, 96, binding.KDA_BF16, 0), (1, 1000, H, 128, 64, binding.KDA_F32, 0),
                (0, 1000, H, d, d, binding.KDA_BF16, 0), (1, 1000, H, d, d, 7, 0)):
        assert lib.kda_prefill_host_workspace_bytes(*bad) == 0


def _hargs(**kw):
    base = dict(q=16, k=32, v=48, g=64, beta=80, state_in=None, B=1, T=100, H=2, dk=64, dv=64,
                dtype=binding.KDA_F32, o=96, state_out=None, segment=0, workspace=None,
                workspace_bytes=0)
    base.update(kw)
    return base


@pytest.mark.parametrize("bad,code", [
    (dict(B=-1), "KDA_ERR_INVALID_ARG"), (dict(T=-5), "KDA_ERR_INVALID_ARG"),
    (dict(H=0), "KDA_ERR_INVALID_ARG"), (dict(dtype=4), "KDA_ERR_INVALID_ARG"),
    (dict(segment=-64), "KDA_ERR_INVALID_ARG"), (dict(q=None), "KDA_ERR_INVALID_ARG"),
    (dict(beta=None), "KDA_ERR_INVALID_ARG"), (dict(o=None), "KDA_ERR_INVALID_ARG"),
    (dict(dk=96, dv=96), "KDA_ERR_UNSUPPORTED"), (dict(dk=128), "KDA_ERR_UNSUPPORTED"),
    (dict(segment=96), "KDA_ERR_UNSUPPORTED"),
    (dict(), "KDA_ERR_INVALID_ARG"),                                   # no workspace
    (dict(workspace=256, workspace_bytes=1024), "KDA_ERR_INVALID_ARG"),    # short workspace
    (dict(workspace=128, workspace_bytes=1 << 40), "KDA_ERR_INVALID_ARG")])  # misaligned
def test_host_prefill_rejects(lib, bad, code):
    assert binding.raw_prefill_host(_hargs(**bad)) == getattr(binding, code)


def test_host_prefill_empty_is_a_no_op(lib):
    assert binding.raw_prefill_host(_hargs(B=0)) == binding.KDA_OK
    assert binding.raw_prefill_host(_hargs(T=0)) == binding.KDA_OK
