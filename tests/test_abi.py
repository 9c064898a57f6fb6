"""The C ABI library on the host (no GPU): it loads, exports every symbol that
include/attn.h declares, and rejects bad arguments before touching CUDA."""

import ctypes
import os
import subprocess

import pytest

from exact_attention_150_b200 import build, native

FAKE = 0x10000  # 16-byte aligned; never dereferenced: every case below fails validation first


@pytest.fixture(scope="module")
def lib():
    build.build()
    return native.load()


def test_header_declares_the_boundary():
    names = set(native.declared_symbols())
    assert {"attn_fwd", "attn_bwd", "attn_bwd_phase", "attn_bwd_workspace_bytes", "attn_last_device_status",
            "attn_status_string", "attn_bwd_deterministic"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in native.declared_symbols():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", native.LIB_PATH], capture_output=True, text=True, check=True)
    exported = {line.split()[-1] for line in out.stdout.splitlines() if line.strip()}
    for name in native.declared_symbols():
        assert name in exported, name


def test_library_is_built_for_sm100a(lib):
    out = subprocess.run(["cuobjdump", "--list-elf", native.LIB_PATH], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    assert "sm_100a" in out.stdout


def test_status_strings(lib):
    assert native.status_string(0) == "ok"
    for s in range(1, 5):
        assert native.status_string(s) not in ("ok", "")
    assert native.status_string(99) == "unknown status"


def _fwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, Nq=128, Nk=128, d=64, scale=0.125, causal=0,
                dtype=native.ATTN_BF16, stream=None)
    args.update(kw)
    return native.attn_fwd(**args)


def _bwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, workspace=FAKE,
                B=1, H=1, Nq=128, Nk=128, d=64, scale=0.125, causal=0, dtype=native.ATTN_FP16, stream=None)
    args.update(kw)
    return native.attn_bwd(**args)


@pytest.mark.parametrize("field", ["q", "k", "v", "o", "lse"])
def test_fwd_null_pointer(lib, field):
    assert _fwd(**{field: None}) == native.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("field", ["q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv", "workspace"])
def test_bwd_null_and_misaligned_pointer(lib, field):
    assert _bwd(**{field: None}) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(**{field: FAKE + 8}) == native.ATTN_ERR_INVALID_ARG


def test_fwd_misaligned_pointer(lib):
    assert _fwd(q=FAKE + 2) == native.ATTN_ERR_INVALID_ARG
    assert _fwd(lse=FAKE + 4) == native.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("field", ["B", "H", "Nq", "Nk", "d"])
def test_negative_sizes(lib, field):
    assert _fwd(**{field: -128}) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(**{field: -128}) == native.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("field", ["B", "H", "Nq"])
def test_empty_problem_is_a_no_op(lib, field):
    """No query rows (or no batch/heads): nothing to write, so success without
    touching any pointer or the device."""
    nulls = dict(q=None, k=None, v=None, o=None, lse=None)
    assert _fwd(**{field: 0}, **nulls) == native.ATTN_OK
    if field != "Nq":  # Nq == 0 with keys still writes dK = dV = 0 (a device memset)
        assert _bwd(**{field: 0}, **nulls, dout=None, dq=None, dk=None, dv=None, workspace=None) == native.ATTN_OK


def test_no_keys_is_invalid(lib):
    assert _fwd(Nk=0) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(Nk=0) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(Nk=0, Nq=0) == native.ATTN_OK


@pytest.mark.parametrize("kw", [dict(d=96), dict(d=512), dict(d=32), dict(d=0), dict(dtype=2), dict(dtype=-1),
                                dict(Nq=65535 * 128 + 1), dict(Nk=65535 * 128 + 1),
                                # B*H times the tile count exceeds the one-dimensional grid
                                dict(B=1 << 16, H=1 << 10, Nq=64 * 128), dict(B=1 << 16, H=1 << 10, Nk=64 * 128)])
def test_unsupported_shapes(lib, kw):
    assert _fwd(**kw) == native.ATTN_ERR_UNSUPPORTED
    assert _bwd(**kw) == native.ATTN_ERR_UNSUPPORTED


def _ws_expected(BH, Nq, d):
    # dQ accumulator padded to whole 128-row query tiles, D and -log2(e) LSE,
    # then (16-byte aligned) one int32 order counter per (b*h, query tile).
    tiles = -(-Nq // 128)
    words = (BH * Nq + tiles * 128 - Nq) * d + 2 * BH * Nq
    words = -(-words // 4) * 4
    return 4 * (words + BH * tiles)


def test_workspace_size(lib):
    assert native.attn_bwd_workspace_bytes(2, 16, 4096, 4096, 64) == 4 * 2 * 16 * 4096 * (64 + 2) + 4 * 32 * 32
    assert native.attn_bwd_workspace_bytes(1, 16, 16384, 16384, 128) == 4 * 16 * 16384 * 130 + 4 * 16 * 128
    assert native.attn_bwd_workspace_bytes(0, 1, 128, 128, 64) == 0
    assert native.attn_bwd_workspace_bytes(1, 1, -1, 128, 64) == 0
    # A ragged last query tile pads the dQ accumulator to a whole tile.
    assert native.attn_bwd_workspace_bytes(2, 3, 300, 77, 64) == _ws_expected(6, 300, 64)
    assert native.attn_bwd_workspace_bytes(2, 3, 300, 77, 64) >= 4 * ((6 * 300 + 84) * 64 + 2 * 6 * 300)
    assert native.attn_bwd_workspace_bytes(1, 1, 1, 1, 128) == _ws_expected(1, 1, 128)
    assert native.attn_bwd_workspace_bytes(3, 1, 5, 9, 64) == _ws_expected(3, 5, 64)


@pytest.mark.parametrize("field", ["q", "dq", "workspace"])
def test_deterministic_bwd_validates_like_bwd(lib, field):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, workspace=FAKE,
                B=1, H=1, Nq=128, Nk=128, d=64, scale=0.125, causal=0, dtype=native.ATTN_FP16, stream=None)
    assert native.attn_bwd_deterministic(**{**args, field: None}) == native.ATTN_ERR_INVALID_ARG
    assert native.attn_bwd_deterministic(**{**args, "d": 96}) == native.ATTN_ERR_UNSUPPORTED
    assert native.attn_bwd_deterministic(**{**args, "causal": 5}) == native.ATTN_ERR_INVALID_ARG
    assert native.attn_bwd_deterministic(**{**args, "B": 0}) == native.ATTN_OK


def test_tensor_wrapper_rejects_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        native.forward(q, q, q)
    with pytest.raises(TypeError):
        native.forward(q.float(), q.float(), q.float())


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(native, "_lib", None)
    monkeypatch.setattr(native, "LIB_PATH", str(tmp_path / "libattn.so"))
    with pytest.raises(RuntimeError, match="missing"):
        native.load()


@pytest.mark.parametrize("phase", [-1, 4, 99])
def test_bwd_phase_out_of_range(lib, phase):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, workspace=FAKE,
                B=1, H=1, Nq=128, Nk=128, d=64, scale=0.125, causal=0, dtype=native.ATTN_FP16, phase=phase,
                stream=None)
    assert native.attn_bwd_phase(**args) == native.ATTN_ERR_INVALID_ARG


def test_bwd_phase_validates_like_bwd(lib):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, workspace=FAKE,
                B=1, H=1, Nq=128, Nk=128, d=96, scale=0.125, causal=0, dtype=native.ATTN_FP16,
                phase=native.ATTN_BWD_MAIN, stream=None)
    assert native.attn_bwd_phase(**args) == native.ATTN_ERR_UNSUPPORTED
    args.update(d=64, dq=None)
    assert native.attn_bwd_phase(**args) == native.ATTN_ERR_INVALID_ARG
    args.update(B=0)
    assert native.attn_bwd_phase(**args) == native.ATTN_OK


@pytest.mark.parametrize("causal", [-1, 3, 99])
def test_causal_value_out_of_range(lib, causal):
    assert _fwd(causal=causal) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(causal=causal) == native.ATTN_ERR_INVALID_ARG
    assert _fwd(causal=causal, B=0) == native.ATTN_ERR_INVALID_ARG  # validated before the empty-problem exit


def test_causal_codes_match_the_header():
    import re
    text = open(native.HEADER).read()
    values = {m.group(1): int(m.group(2)) for m in re.finditer(r"(ATTN_CAUSAL_\w+)\s*=\s*(\d+)", text)}
    assert values == {"ATTN_CAUSAL_NONE": native.ATTN_CAUSAL_NONE, "ATTN_CAUSAL_TOP_LEFT": native.ATTN_CAUSAL_TOP_LEFT,
                      "ATTN_CAUSAL_BOTTOM_RIGHT": native.ATTN_CAUSAL_BOTTOM_RIGHT}
    assert [native.causal_code(c) for c in (False, True, "none", "top_left", "bottom_right", 2)] == [0, 1, 0, 1, 2, 2]
    with pytest.raises(ValueError):
        native.causal_code("bottom-left")


def _fwd_varlen(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cu_q=FAKE, cu_k=FAKE, B=2, H=3, total_q=300, total_k=400,
                max_q=200, max_k=300, d=64, scale=0.125, causal=0, dtype=native.ATTN_BF16, stream=None)
    args.update(kw)
    return native.attn_fwd_varlen(**args)


def _bwd_varlen(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, workspace=FAKE,
                cu_q=FAKE, cu_k=FAKE, B=2, H=3, total_q=300, total_k=400, max_q=200, max_k=300, d=64, scale=0.125,
                causal=0, dtype=native.ATTN_BF16, deterministic=0, stream=None)
    args.update(kw)
    return native.attn_bwd_varlen(**args)


@pytest.mark.parametrize("fn", [_fwd_varlen, _bwd_varlen])
def test_varlen_validation(lib, fn):
    for field in ("B", "H", "total_q", "total_k", "max_q", "max_k"):
        assert fn(**{field: -1}) == native.ATTN_ERR_INVALID_ARG
    assert fn(d=96) == native.ATTN_ERR_UNSUPPORTED
    assert fn(dtype=5) == native.ATTN_ERR_UNSUPPORTED
    assert fn(causal=3) == native.ATTN_ERR_INVALID_ARG
    assert fn(max_q=65535 * 128 + 1) == native.ATTN_ERR_UNSUPPORTED
    assert fn(B=1 << 16, H=1 << 10, max_q=64 * 128) == native.ATTN_ERR_UNSUPPORTED
    assert fn(B=1 << 16, H=1 << 10, max_k=64 * 128) == native.ATTN_ERR_UNSUPPORTED
    assert fn(cu_q=None) == native.ATTN_ERR_INVALID_ARG
    assert fn(cu_k=FAKE + 2) == native.ATTN_ERR_INVALID_ARG  # offsets must be 4-byte aligned
    assert fn(q=FAKE + 8) == native.ATTN_ERR_INVALID_ARG
    assert fn(B=0) == native.ATTN_OK
    assert fn(H=0) == native.ATTN_OK


def test_varlen_workspace_size(lib):
    for B, H, total_q, max_q, d in ((2, 3, 300, 200, 64), (5, 16, 4096, 1024, 128), (1, 1, 1, 1, 128)):
        tiles = -(-max_q // 128)
        rows = H * total_q
        words = (rows + 128) * d + 2 * rows
        words = -(-words // 4) * 4 + B * H * tiles
        assert native.attn_bwd_varlen_workspace_bytes(B, H, total_q, max_q, d) == 4 * words
    assert native.attn_bwd_varlen_workspace_bytes(0, 3, 300, 200, 64) == 0


@pytest.mark.parametrize("limit_us", [0, -5, 1000001])
def test_selftest_rejects_bad_limits(lib, limit_us):
    assert native.load().attn_selftest_wait_timeout(limit_us, FAKE, None) == native.ATTN_ERR_INVALID_ARG


def test_selftest_rejects_null_result(lib):
    assert native.load().attn_selftest_wait_timeout(1000, None, None) == native.ATTN_ERR_INVALID_ARG


def test_head_dim_256_is_validated_like_any_supported_d(lib):
    """d = 256 passes every entry point's shape checks: a NULL pointer is then
    what gets refused (nothing is launched with the fake pointers)."""
    assert _bwd(d=256, q=None) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(d=256, Nq=0, dq=None, dout=None, q=None, o=None, lse=None, dk=None) == native.ATTN_ERR_INVALID_ARG
    assert _bwd_varlen(d=256, q=None) == native.ATTN_ERR_INVALID_ARG
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, workspace=None,
                B=1, H=1, Nq=128, Nk=128, d=256, scale=0.1, causal=0, dtype=native.ATTN_BF16, stream=None)
    assert native.attn_bwd_deterministic(**args) == native.ATTN_ERR_INVALID_ARG
    assert _fwd(d=256, q=None) == native.ATTN_ERR_INVALID_ARG
    assert _bwd(d=96, q=None) == native.ATTN_ERR_UNSUPPORTED


def _fwd_fp8(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, Nq=128, Nk=128, d=128, scale=0.125,
                descale_q=1.0, descale_k=1.0, descale_v=1.0, causal=0, stream=None)
    args.update(kw)
    return native.attn_fwd_fp8(**args)


def test_fp8_forward_validation(lib):
    for d in (64, 96, 256, 0):
        assert _fwd_fp8(d=d) == native.ATTN_ERR_UNSUPPORTED
    for field in ("descale_q", "descale_k", "descale_v", "scale"):
        assert _fwd_fp8(**{field: float("nan")}) == native.ATTN_ERR_INVALID_ARG
        assert _fwd_fp8(**{field: float("inf")}) == native.ATTN_ERR_INVALID_ARG
    for field in ("B", "H", "Nq", "Nk"):
        assert _fwd_fp8(**{field: -1}) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8(causal=3) == native.ATTN_ERR_INVALID_ARG
    for name in ("q", "k", "v", "o", "lse"):
        assert _fwd_fp8(**{name: None}) == native.ATTN_ERR_INVALID_ARG
        assert _fwd_fp8(**{name: FAKE + 8}) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8(Nk=0) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8(Nq=65535 * 128 + 1) == native.ATTN_ERR_UNSUPPORTED
    assert _fwd_fp8(B=1 << 16, H=1 << 10, Nq=64 * 128) == native.ATTN_ERR_UNSUPPORTED
    # Empty problems are valid and touch nothing.
    assert _fwd_fp8(B=0, q=None, k=None, v=None, o=None, lse=None) == native.ATTN_OK
    assert _fwd_fp8(Nq=0, q=None, k=None, v=None, o=None, lse=None) == native.ATTN_OK


def _host_step(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, dout=FAKE, o=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
                device_buffer=FAKE, device_bytes=1 << 40, B=1, H=4, Nq=300, Nk=300, d=128, scale=0.1, causal=1,
                dtype=native.ATTN_BF16, chunks=2, deterministic=0, stream=None)
    args.update(kw)
    return native.attn_host_step(**args)


def _host_step_bytes(B, H, Nq, Nk, d, chunks):
    # Every region rounded up to 256 bytes: Q, K, V, dO, O, dQ, dK, dV, then
    # one aligned LSE block per chunk, then one chunk's backward workspace.
    r = lambda x: (x + 255) // 256 * 256
    bh = B * H
    chunks = min(chunks, bh)
    per = -(-bh // chunks)
    chunks = -(-bh // per)
    qb, kb = r(bh * Nq * d * 2), r(bh * Nk * d * 2)
    return 4 * qb + 4 * kb + r(r(per * Nq * 4) * chunks) + r(native.attn_bwd_workspace_bytes(1, per, Nq, Nk, d))


@pytest.mark.parametrize("shape", [(1, 16, 16384, 16384, 128, 4), (2, 3, 300, 129, 64, 4), (1, 5, 7, 9, 128, 3),
                                   (3, 1, 128, 128, 64, 1), (2, 2, 100, 200, 128, 9)])
def test_host_step_device_bytes(lib, shape):
    assert native.attn_host_step_device_bytes(*shape) == _host_step_bytes(*shape)


def test_host_step_device_bytes_empty(lib):
    assert native.attn_host_step_device_bytes(0, 4, 128, 128, 128, 2) == 0
    assert native.attn_host_step_device_bytes(1, 4, 0, 128, 128, 2) == 0
    assert native.attn_host_step_device_bytes(1, 4, 128, 128, 128, 0) == 0
    # Past the attention calls' row bounds (B*H*N <= 2^40): no size, rather than a wrapped one.
    assert native.attn_host_step_device_bytes(1 << 16, 1 << 14, 1, (1 << 23) - 1, 128, 4) == 0


def test_host_step_validation(lib):
    assert _host_step(chunks=0) == native.ATTN_ERR_INVALID_ARG
    for d in (96, 0):
        assert _host_step(d=d) == native.ATTN_ERR_UNSUPPORTED
    assert _host_step(d=256, q=None) == native.ATTN_ERR_INVALID_ARG  # a supported d: checked further
    assert _host_step(dtype=5) == native.ATTN_ERR_UNSUPPORTED
    assert _host_step(causal=3) == native.ATTN_ERR_INVALID_ARG
    for field in ("B", "H", "Nq", "Nk"):
        assert _host_step(**{field: -1}) == native.ATTN_ERR_INVALID_ARG
    for name in ("q", "k", "v", "dout", "o", "lse", "dq", "dk", "dv", "device_buffer"):
        assert _host_step(**{name: None}) == native.ATTN_ERR_INVALID_ARG
    assert _host_step(device_buffer=FAKE + 16) == native.ATTN_ERR_INVALID_ARG  # 256-byte alignment
    need = native.attn_host_step_device_bytes(1, 4, 300, 300, 128, 2)
    assert _host_step(device_bytes=need - 1) == native.ATTN_ERR_INVALID_ARG
    assert _host_step(Nk=0) == native.ATTN_ERR_INVALID_ARG
    assert _host_step(B=1 << 16, H=1 << 16) == native.ATTN_ERR_UNSUPPORTED
    assert _host_step(B=0) == native.ATTN_OK  # nothing to do
    assert _host_step(Nq=0, Nk=0) == native.ATTN_OK


def _fwd_fp8_varlen(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cu_q=FAKE, cu_k=FAKE, B=2, H=3, total_q=300, total_k=400,
                max_q=200, max_k=300, d=128, scale=0.125, descale_q=1.0, descale_k=1.0, descale_v=1.0, causal=0,
                stream=None)
    args.update(kw)
    return native.attn_fwd_fp8_varlen(**args)


def test_fp8_varlen_validation(lib):
    for field in ("B", "H", "total_q", "total_k", "max_q", "max_k"):
        assert _fwd_fp8_varlen(**{field: -1}) == native.ATTN_ERR_INVALID_ARG
    for d in (64, 256, 96):
        assert _fwd_fp8_varlen(d=d) == native.ATTN_ERR_UNSUPPORTED
    for field in ("descale_q", "descale_k", "descale_v", "scale"):
        assert _fwd_fp8_varlen(**{field: float("nan")}) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(causal=3) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(max_q=65535 * 128 + 1) == native.ATTN_ERR_UNSUPPORTED
    for name in ("q", "k", "v", "o", "lse", "cu_q", "cu_k"):
        assert _fwd_fp8_varlen(**{name: None}) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(cu_k=FAKE + 2) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(q=FAKE + 8) == native.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(B=0) == native.ATTN_OK
    assert _fwd_fp8_varlen(total_q=0) == native.ATTN_OK
