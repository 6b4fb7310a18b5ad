"""The C-ABI library loads and exports every function include/h3dit.h declares;
host-side argument checks return their status codes. No compute call is made,
so these run without a GPU."""
import ctypes as C
import subprocess

import pytest

from image_generation_b200 import h3dit as H


def test_library_exports_every_declared_function():
    declared = H.header_functions()
    assert "h3dit_create" in declared and "h3dit_step" in declared
    out = subprocess.run(["nm", "-D", "--defined-only", H.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for f in declared:
        assert hasattr(H.lib, f)


def test_profile_kinds_match_the_header():
    """The binding names one profile slot per H3DIT_KERNEL_* value, in order."""
    import re

    with open(H.HEADER) as fh:
        text = fh.read()
    kinds = {m.group(1): int(m.group(2))
             for m in re.finditer(r"#define H3DIT_KERNEL_([A-Z_0-9]+)\s+(\d+)", text)}
    count = kinds.pop("COUNT")
    assert count == len(H.KERNEL_KINDS)
    assert sorted(kinds.values()) == list(range(count))
    by_value = {v: k.lower() for k, v in kinds.items()}
    assert [by_value[i] for i in range(count)] == H.KERNEL_KINDS


def test_status_strings():
    for s in (H.H3DIT_OK, H.H3DIT_ERR_INVALID_ARG, H.H3DIT_ERR_UNSUPPORTED,
              H.H3DIT_ERR_WORKSPACE, H.H3DIT_ERR_CUDA, H.H3DIT_ERR_TIMEOUT):
        assert H.status_string(s) and H.status_string(s) != "unknown status"
    assert H.status_string(12345) == "unknown status"


def _cfg(**kw):
    base = dict(hidden=5376, heads=56, head_dim=96, ffn=14336, n_blocks=50, max_tokens=16896)
    base.update(kw)
    return H.make_config(**base)


def test_workspace_bytes_covers_the_plan():
    cfg = _cfg()
    ws = H.lib.h3dit_workspace_bytes(C.byref(cfg))
    N, D, I, F, L = 16896, 5376, 5376, 14336, 50
    need = N * D * 4 + N * D * 2 + N * 3 * I * 2 + N * I * 2 + N * F * 2 + L * 6 * D * 4
    assert need <= ws <= need + 64 * 1024 * 1024
    # head_dim 128 makes the attention width 7168
    ws128 = H.lib.h3dit_workspace_bytes(C.byref(_cfg(head_dim=128)))
    assert ws128 > ws


@pytest.mark.parametrize("bad", [
    dict(hidden=100), dict(head_dim=64), dict(ffn=1000), dict(n_blocks=0), dict(max_tokens=0),
    dict(sections=(16, 16, 8)), dict(heads=0),
])
def test_invalid_configs_have_no_workspace(bad):
    assert H.lib.h3dit_workspace_bytes(C.byref(_cfg(**bad))) == 0
    assert H.lib.h3dit_workspace_bytes(None) == 0


def _fake_weights(n_blocks):
    fake = 0x10000  # 16-byte aligned, never dereferenced by the host-side checks
    tw = H.h3dit_time_weights(fake, fake, fake, fake)
    arr = (H.h3dit_block_weights * n_blocks)()
    for i in range(n_blocks):
        arr[i] = H.h3dit_block_weights(fake, fake, fake, fake, fake, fake)
    return tw, arr


def test_create_rejects_bad_arguments_before_touching_the_device():
    cfg = _cfg(hidden=768, heads=8, ffn=2048, n_blocks=2, max_tokens=288)
    tw, arr = _fake_weights(2)
    out = C.c_void_p(1)
    ws = H.lib.h3dit_workspace_bytes(C.byref(cfg))
    # no workspace
    assert H.lib.h3dit_create(C.byref(cfg), C.byref(tw), arr, None, ws, None, C.byref(out)) \
        == H.H3DIT_ERR_WORKSPACE
    assert out.value is None
    # too small / misaligned workspace
    assert H.lib.h3dit_create(C.byref(cfg), C.byref(tw), arr, 0x100000, ws - 1, None,
                              C.byref(out)) == H.H3DIT_ERR_WORKSPACE
    assert H.lib.h3dit_create(C.byref(cfg), C.byref(tw), arr, 0x100010, ws, None,
                              C.byref(out)) == H.H3DIT_ERR_WORKSPACE
    # NULL weights, misaligned weight, bad config, NULL out
    assert H.lib.h3dit_create(C.byref(cfg), None, arr, 0x100000, ws, None, C.byref(out)) \
        == H.H3DIT_ERR_INVALID_ARG
    arr[1].w_o = 0x10002
    assert H.lib.h3dit_create(C.byref(cfg), C.byref(tw), arr, 0x100000, ws, None,
                              C.byref(out)) == H.H3DIT_ERR_INVALID_ARG
    bad = _cfg(hidden=100)
    assert H.lib.h3dit_create(C.byref(bad), C.byref(tw), arr, 0x100000, ws, None,
                              C.byref(out)) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_create(C.byref(cfg), C.byref(tw), arr, 0x100000, ws, None, None) \
        == H.H3DIT_ERR_INVALID_ARG
    # MXFP8 with a width that is not a multiple of 128 is not run
    mx = _cfg(hidden=832, heads=8, ffn=2048, n_blocks=2, max_tokens=288, precision=1)
    tw, arr = _fake_weights(2)
    assert H.lib.h3dit_create(C.byref(mx), C.byref(tw), arr, 0x100000, ws, None,
                              C.byref(out)) == H.H3DIT_ERR_UNSUPPORTED
    # the MXFP8 workspace also holds the quantized weights
    mx_ok = _cfg(hidden=768, heads=8, ffn=2048, n_blocks=2, max_tokens=288, precision=1)
    assert H.lib.h3dit_workspace_bytes(C.byref(mx_ok)) > ws + 2 * (4 * 768 * 768 + 2 * 768 * 2048)


def test_null_context_is_rejected_everywhere():
    g = H.grids_array([(0, 2, 2)])
    assert H.lib.h3dit_block_forward(None, 0, 0.5, None, 0x10000, g, 1, None, 0, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_step(None, 0.5, 0x10000, g, 1, None, 0, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_sync_status(None, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_time_embed(None, 0.5, 0x10000, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_adaln_project(None, 0x10000, 0, 1, 0x10000, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_rmsnorm_modulate(None, 0x10000, 0x10000, 0x10000, 0x10000, 4, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_rope_table(None, g, 1, 0, 0x10000, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_linear(None, 0, 0x10000, 0x10000, 4, 32, 64, 0x10000, None, None, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_attention(None, 0x10000, 0x10000, 0x10000, 768, 0x10000, 768, 4, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_block_linear_mx(None, 0, H.H3DIT_LINEAR_QKV, 0x10000, 0x10000, 4, 0x10000,
                                       None, None, 0x10000, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_embed_latent(None, 0x10000, 24, 4, 4, 0x10000, 0x10000, 0x10000, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_output_modulation(None, 0x10000, 0x10000, 0x10000, 0x10000, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_output_euler(None, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 24, 4, 4,
                                    -0.1, None) == H.H3DIT_ERR_INVALID_ARG
    io = H.h3dit_io_weights(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    assert H.lib.h3dit_denoise(None, C.byref(io), 0x10000, 24, 4, 4, 0x10000, 8, 6, None) \
        == H.H3DIT_ERR_INVALID_ARG
    dst = (C.c_void_p * 2)(0x10000, 0x20000)
    assert H.lib.h3dit_sp_qkv_scatter(None, 0x10000, 4, 0x10000, 0x10000, dst, 2, 0, None) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_sp_attention_scatter(None, 0x10000, 8, dst, 2, 0, None) \
        == H.H3DIT_ERR_INVALID_ARG
    H.lib.h3dit_destroy(None)  # NULL-safe
    assert H.lib.h3dit_last_error(None) == b"no context"


def test_ipc_calls_reject_null_arguments_before_the_runtime():
    off = C.c_uint64()
    ptr = C.c_void_p()
    handle = bytes(H.H3DIT_IPC_HANDLE_BYTES)
    assert H.lib.h3dit_ipc_get_handle(None, handle, C.byref(off)) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_ipc_get_handle(0x10000, None, C.byref(off)) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_ipc_get_handle(0x10000, handle, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_ipc_open(None, 0, C.byref(ptr)) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_ipc_open(handle, 0, None) == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_ipc_close(None, 0) == H.H3DIT_ERR_INVALID_ARG
    with pytest.raises(H.H3DitError):
        H.ipc_open(b"short", 0)  # the binding checks the handle's size


def test_mx_scale_layout_size():
    assert H.mx_scale_bytes(128, 128) == 512
    assert H.mx_scale_bytes(129, 256) == 2 * 2 * 512
    assert H.mx_scale_bytes(16896, 5376) == 132 * 42 * 512
    assert H.mx_scale_bytes(100, 96) == 0
    # every (row, block) of a matrix lands on a distinct byte of the array
    rows, k = 256, 384
    offs = {H.mx_sf_offset(r, s, k) for r in range(rows) for s in range(k // 32)}
    assert len(offs) == rows * k // 32 and max(offs) < H.mx_scale_bytes(rows, k)


def test_binding_rejects_host_tensors_before_the_library_sees_them():
    """Tensor arguments go to the kernels as device addresses, so a host tensor
    is refused in the binding (the library cannot tell a host address apart)."""
    import torch

    assert H._ptr(None) is None
    for dense in (True, False):
        with pytest.raises(H.H3DitError) as e:
            H._ptr(torch.zeros(4), dense)
        assert e.value.status == H.H3DIT_ERR_INVALID_ARG
