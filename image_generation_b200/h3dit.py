"""ctypes binding of libh3dit (include/h3dit.h), same names as the C ABI.

Argument marshalling only: every step of the block runs in the CUDA kernels of
libh3dit.so. There is no fallback: if the library is missing, importing the
binding raises. PyTorch is used by the helpers at the bottom only to hold
device memory and to name the current CUDA stream.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import List, Sequence, Tuple

PKG = os.path.dirname(os.path.abspath(__file__))
# H3DIT_LIB selects another build of the library (the stamped diagnostic
# build); the product library is the default.
LIB_PATH = os.environ.get("H3DIT_LIB") or os.path.join(PKG, "libh3dit.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "h3dit.h")

H3DIT_OK = 0
H3DIT_ERR_INVALID_ARG = -1
H3DIT_ERR_UNSUPPORTED = -2
H3DIT_ERR_WORKSPACE = -3
H3DIT_ERR_CUDA = -4
H3DIT_ERR_TIMEOUT = -5

H3DIT_EPI_STORE = 0
H3DIT_EPI_QKV_ROPE = 1
H3DIT_EPI_GELU = 2
H3DIT_EPI_GATED_RESIDUAL = 3

H3DIT_LINEAR_QKV = 0
H3DIT_LINEAR_OUT = 1
H3DIT_LINEAR_FFN1 = 2
H3DIT_LINEAR_FFN2 = 3

H3DIT_PRECISION_BF16 = 0
H3DIT_PRECISION_MXFP8 = 1
H3DIT_STATIC_TIME_MAX_HIDDEN = 8192
H3DIT_MAX_SCATTER_RANKS = 8
H3DIT_IPC_HANDLE_BYTES = 64
H3DIT_ATTN_STAMP_SLOTS = 32
H3DIT_ATTN_STAMP_STEPS = 300

KERNEL_KINDS = ["time_embed", "adaln", "rmsnorm", "qkv", "attention", "out_proj", "ffn1",
                "ffn2", "rope_table", "pack", "mx_quantize", "io"]


class h3dit_config(C.Structure):
    _fields_ = [
        ("hidden", C.c_int32), ("heads", C.c_int32), ("head_dim", C.c_int32),
        ("ffn", C.c_int32), ("n_blocks", C.c_int32), ("max_tokens", C.c_int32),
        ("rope_sections", C.c_int32 * 3), ("rope_theta", C.c_float),
        ("norm_eps", C.c_float), ("t_scale", C.c_float), ("gelu_tanh", C.c_int32),
        ("precision", C.c_int32), ("io_fp32", C.c_int32),
    ]


class h3dit_time_weights(C.Structure):
    _fields_ = [("w_t1", C.c_void_p), ("b_t1", C.c_void_p), ("w_t2", C.c_void_p),
                ("b_t2", C.c_void_p)]


class h3dit_block_weights(C.Structure):
    _fields_ = [("w_qkv", C.c_void_p), ("w_o", C.c_void_p), ("w_ff1", C.c_void_p),
                ("w_ff2", C.c_void_p), ("w_ada", C.c_void_p), ("b_ada", C.c_void_p)]


class h3dit_io_weights(C.Structure):
    _fields_ = [("w_in", C.c_void_p), ("b_in", C.c_void_p), ("w_mod", C.c_void_p),
                ("b_mod", C.c_void_p), ("w_out", C.c_void_p), ("b_out", C.c_void_p)]


class h3dit_vae_config(C.Structure):
    _fields_ = [("width", C.c_int32), ("heads", C.c_int32), ("head_dim", C.c_int32),
                ("mlp", C.c_int32), ("layers", C.c_int32), ("tile", C.c_int32),
                ("channels", C.c_int32), ("max_tokens", C.c_int32), ("eps", C.c_float)]


class h3dit_vae_layer_weights(C.Structure):
    _fields_ = [(k, C.c_void_p) for k in ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                                           "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")]


class h3dit_vae_weights(C.Structure):
    _fields_ = [("w_in", C.c_void_p), ("b_in", C.c_void_p),
                ("layers", C.POINTER(h3dit_vae_layer_weights)), ("lnf_g", C.c_void_p),
                ("lnf_b", C.c_void_p), ("w_out", C.c_void_p), ("b_out", C.c_void_p)]


class h3dit_grid(C.Structure):
    _fields_ = [("frame", C.c_int32), ("height", C.c_int32), ("width", C.c_int32)]


class H3DitError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"h3dit status {status}: {msg}")
        self.status = status


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m image_generation_b200.build`")
    lib = C.CDLL(LIB_PATH)
    p, i32, f32, sz = C.c_void_p, C.c_int32, C.c_float, C.c_size_t
    sig = {
        "h3dit_status_string": (C.c_char_p, [i32]),
        "h3dit_last_error": (C.c_char_p, [p]),
        "h3dit_workspace_bytes": (sz, [C.POINTER(h3dit_config)]),
        "h3dit_create": (i32, [C.POINTER(h3dit_config), C.POINTER(h3dit_time_weights),
                               C.POINTER(h3dit_block_weights), p, sz, p, C.POINTER(p)]),
        "h3dit_destroy": (None, [p]),
        "h3dit_block_forward": (i32, [p, i32, f32, p, p, C.POINTER(h3dit_grid), i32, p, i32, p]),
        "h3dit_step": (i32, [p, f32, p, C.POINTER(h3dit_grid), i32, p, i32, p]),
        "h3dit_sync_status": (i32, [p, p]),
        "h3dit_time_embed": (i32, [p, f32, p, p]),
        "h3dit_adaln_project": (i32, [p, p, i32, i32, p, p]),
        "h3dit_rmsnorm_modulate": (i32, [p, p, p, p, p, i32, p]),
        "h3dit_rope_table": (i32, [p, C.POINTER(h3dit_grid), i32, i32, p, p]),
        "h3dit_linear": (i32, [p, i32, p, p, i32, i32, i32, p, p, p, p]),
        "h3dit_attention": (i32, [p, p, p, p, i32, p, i32, i32, p]),
        "h3dit_time_embed_static": (i32, [p, p, p, p, i32, f32, f32, p, p]),
        "h3dit_mx_scale_bytes": (sz, [i32, i32]),
        "h3dit_mx_quantize": (i32, [p, p, i32, i32, p, p, p]),
        "h3dit_linear_mx": (i32, [p, i32, p, p, p, p, i32, i32, i32, p, p, p, p, p]),
        "h3dit_block_linear_mx": (i32, [p, i32, i32, p, p, i32, p, p, p, p, p]),
        "h3dit_rmsnorm_modulate_mx": (i32, [p, p, p, p, p, p, i32, p]),
        "h3dit_attention_mx": (i32, [p, p, p, p, i32, p, p, i32, p]),
        "h3dit_embed_latent": (i32, [p, p, i32, i32, i32, p, p, p, p]),
        "h3dit_output_modulation": (i32, [p, p, p, p, p, p]),
        "h3dit_output_euler": (i32, [p, p, p, p, p, p, i32, i32, i32, f32, p]),
        "h3dit_denoise": (i32, [p, C.POINTER(h3dit_io_weights), p, i32, i32, i32, p, i32, i32,
                                p]),
        "h3dit_attention_heads": (i32, [p, i32, p, p, p, i32, p, i32, i32, p]),
        "h3dit_sp_pack_qkv": (i32, [p, p, i32, i32, p, p]),
        "h3dit_sp_unpack_o": (i32, [p, p, i32, i32, p, p]),
        "h3dit_sp_qkv_scatter": (i32, [p, p, i32, p, p, C.POINTER(p), i32, i32, p]),
        "h3dit_sp_attention_scatter": (i32, [p, p, i32, C.POINTER(p), i32, i32, p]),
        "h3dit_sp_qkv_scatter_mx": (i32, [p, p, p, i32, i32, p, C.POINTER(p), i32, i32, p]),
        "h3dit_sp_attention_scatter_mx": (i32, [p, p, i32, C.POINTER(p), C.POINTER(p), i32, i32,
                                                p]),
        "h3dit_ipc_get_handle": (i32, [p, p, C.POINTER(C.c_uint64)]),
        "h3dit_ipc_open": (i32, [p, C.c_uint64, C.POINTER(p)]),
        "h3dit_ipc_close": (i32, [p, C.c_uint64]),
        "h3dit_vae_workspace_bytes": (sz, [C.POINTER(h3dit_vae_config)]),
        "h3dit_vae_create": (i32, [C.POINTER(h3dit_vae_config), C.POINTER(h3dit_vae_weights), p,
                                   sz, p, C.POINTER(p)]),
        "h3dit_vae_decode": (i32, [p, p, i32, i32, p, p]),
        "h3dit_layernorm": (i32, [p, p, p, p, p, i32, p]),
        "h3dit_linear_bias": (i32, [p, i32, p, p, p, i32, i32, i32, p, p, p]),
        "h3dit_attention_batched": (i32, [p, p, p, p, i32, p, i32, i32, i32, p]),
        "h3dit_staging_bytes": (sz, [C.POINTER(h3dit_config)]),
        "h3dit_attach_staging": (i32, [p, p, sz, p]),
        "h3dit_streamed_blocks": (i32, [p]),
        "h3dit_selftest_bounded_wait": (i32, [p, i32, p]),
        "h3dit_profile_begin": (i32, [p]),
        "h3dit_profile_end": (i32, [p, C.POINTER(C.c_float), C.POINTER(C.c_int64)]),
        "h3dit_launch_count": (C.c_int64, [p]),
        "h3dit_attention_stamps": (i32, [C.POINTER(C.c_uint64), i32, i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def header_functions() -> List[str]:
    """Names of the functions include/h3dit.h declares."""
    with open(HEADER) as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(h3dit_[a-z_0-9]+)\s*\(", text)))


def status_string(s: int) -> str:
    return lib.h3dit_status_string(s).decode()


def check(ctx, status: int) -> None:
    if status != H3DIT_OK:
        msg = lib.h3dit_last_error(ctx).decode() if ctx else status_string(status)
        raise H3DitError(status, msg or status_string(status))


def make_config(hidden: int, heads: int, head_dim: int, ffn: int, n_blocks: int,
                max_tokens: int, sections: Sequence[int] | None = None,
                rope_theta: float = 10000.0, norm_eps: float = 1e-6, t_scale: float = 1000.0,
                gelu_tanh: bool = False, precision: int = H3DIT_PRECISION_BF16,
                io_fp32: bool = False) -> h3dit_config:
    if sections is None:
        sections = {96: (16, 16, 16), 128: (16, 24, 24)}.get(head_dim, (0, 0, 0))
    return h3dit_config(hidden, heads, head_dim, ffn, n_blocks, max_tokens,
                        (C.c_int32 * 3)(*sections), rope_theta, norm_eps, t_scale,
                        int(gelu_tanh), precision, int(io_fp32))


def mx_scale_bytes(rows: int, k: int) -> int:
    return int(lib.h3dit_mx_scale_bytes(rows, k))


def mx_sf_offset(row: int, s: int, k: int) -> int:
    """Byte of the scale of row `row`, k-block `s` (32 elements) in the layout
    the header documents (for decoding in tests)."""
    return ((row // 128) * (k // 128) + s // 4) * 512 + (row % 32) * 16 + ((row // 32) % 4) * 4 + s % 4


def grids_array(grids: Sequence[Tuple[int, int, int]]):
    arr = (h3dit_grid * max(1, len(grids)))()
    for i, (f, h, w) in enumerate(grids):
        arr[i] = h3dit_grid(f, h, w)
    return arr


# ---------------------------------------------------------------- torch helpers

def _ptr(t, dense: bool = True) -> int | None:
    """Device address of a tensor argument. Every tensor must be on a CUDA
    device. Those the ABI reads as dense arrays must be contiguous; the
    attention operands are strided row views (their row stride is passed
    separately) and only need a unit stride along the last axis."""
    if t is None:
        return None
    if not t.is_cuda:
        raise H3DitError(H3DIT_ERR_INVALID_ARG, "tensor argument is not on a CUDA device")
    if dense and not t.is_contiguous():
        raise H3DitError(H3DIT_ERR_INVALID_ARG, "tensor argument is not contiguous")
    if not dense and t.dim() > 0 and t.stride(-1) != 1:
        raise H3DitError(H3DIT_ERR_INVALID_ARG, "strided operand needs unit stride in its last axis")
    return t.data_ptr()


def _wptr(t) -> int:
    """Address of a block weight: a contiguous CUDA tensor, or a contiguous
    pinned host tensor (a block the library streams to the GPU)."""
    if not t.is_cuda and not t.is_pinned():
        raise H3DitError(H3DIT_ERR_INVALID_ARG, "host weights must be in pinned memory")
    if not t.is_contiguous():
        raise H3DitError(H3DIT_ERR_INVALID_ARG, "tensor argument is not contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def ipc_handle(t) -> Tuple[bytes, int]:
    """(handle, offset) naming the device memory of tensor t for another
    process on this node (CUDA IPC; see h3dit_ipc_get_handle)."""
    h = (C.c_char * H3DIT_IPC_HANDLE_BYTES)()
    off = C.c_uint64()
    check(None, lib.h3dit_ipc_get_handle(_ptr(t, False), h, C.byref(off)))
    return bytes(h), int(off.value)


def ipc_open(handle: bytes, offset: int) -> int:
    """Device address, in this process, of the byte another process named
    with ipc_handle."""
    if len(handle) != H3DIT_IPC_HANDLE_BYTES:
        raise H3DitError(H3DIT_ERR_INVALID_ARG, "IPC handle of the wrong size")
    out = C.c_void_p()
    check(None, lib.h3dit_ipc_open(handle, offset, C.byref(out)))
    return int(out.value)


def ipc_close(ptr: int, offset: int) -> None:
    check(None, lib.h3dit_ipc_close(ptr, offset))


class Context:
    """Owns one h3dit_ctx plus the torch tensors it borrows (weights, workspace)."""

    def __init__(self, cfg: h3dit_config, time_w: dict, blocks: Sequence[dict], stream=None,
                 workspace=None):
        """workspace: optional caller-owned uint8 device tensor of at least
        h3dit_workspace_bytes(cfg) bytes (256-byte aligned); allocated here
        when omitted."""
        import torch

        self.cfg = cfg
        self._keep = [time_w, list(blocks)]
        ws_bytes = lib.h3dit_workspace_bytes(C.byref(cfg))
        if ws_bytes == 0:
            raise H3DitError(H3DIT_ERR_INVALID_ARG, "invalid config")
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        elif workspace.numel() * workspace.element_size() < ws_bytes:
            raise H3DitError(H3DIT_ERR_WORKSPACE, "workspace smaller than h3dit_workspace_bytes")
        self.workspace = workspace
        tw = h3dit_time_weights(_ptr(time_w["w_t1"]), _ptr(time_w["b_t1"]),
                                _ptr(time_w["w_t2"]), _ptr(time_w["b_t2"]))
        arr = (h3dit_block_weights * len(blocks))()
        for i, b in enumerate(blocks):
            arr[i] = h3dit_block_weights(_wptr(b["w_qkv"]), _wptr(b["w_o"]), _wptr(b["w_ff1"]),
                                         _wptr(b["w_ff2"]), _wptr(b["w_ada"]), _wptr(b["b_ada"]))
        handle = C.c_void_p()
        st = lib.h3dit_create(C.byref(cfg), C.byref(tw), arr, _ptr(self.workspace),
                              ws_bytes, _stream(stream), C.byref(handle))
        check(None, st)
        self.handle = handle

    def layernorm(self, x, gain, bias, out, stream=None) -> None:
        self._check(lib.h3dit_layernorm(self.handle, _ptr(x), _ptr(gain), _ptr(bias), _ptr(out),
                                        x.shape[0], _stream(stream)))

    def linear_bias(self, epilogue: int, a, w, bias, out, gate=None, stream=None) -> None:
        m, k = a.shape
        n = w.shape[0]
        self._check(lib.h3dit_linear_bias(self.handle, epilogue, _ptr(a), _ptr(w), _ptr(bias), m,
                                          n, k, _ptr(out), _ptr(gate), _stream(stream)))

    def attention_batched(self, q, k, v, ld_qkv: int, o, ld_o: int, n: int, batch: int,
                          stream=None) -> None:
        self._check(lib.h3dit_attention_batched(self.handle, _ptr(q, False), _ptr(k, False),
                                                _ptr(v, False), ld_qkv, _ptr(o, False), ld_o, n,
                                                batch, _stream(stream)))

    def attach_staging(self, staging=None, copy_stream=None) -> None:
        """Lend the context device staging memory for blocks whose weights are
        in pinned host memory (allocated here when omitted)."""
        import torch

        nbytes = int(lib.h3dit_staging_bytes(C.byref(self.cfg)))
        if staging is None:
            staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.staging = staging
        self._check(lib.h3dit_attach_staging(self.handle, _ptr(staging),
                                             staging.numel() * staging.element_size(),
                                             None if copy_stream is None else copy_stream.cuda_stream))

    def streamed_blocks(self) -> int:
        return int(lib.h3dit_streamed_blocks(self.handle))

    def close(self) -> None:
        if getattr(self, "handle", None):
            lib.h3dit_destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()

    def _check(self, st: int) -> None:
        check(self.handle, st)

    def sync_status(self, stream=None) -> int:
        return lib.h3dit_sync_status(self.handle, _stream(stream))

    def time_embed(self, t: float, c_out, stream=None) -> None:
        self._check(lib.h3dit_time_embed(self.handle, t, _ptr(c_out), _stream(stream)))

    def adaln_project(self, c, first: int, count: int, mod_out, stream=None) -> None:
        self._check(lib.h3dit_adaln_project(self.handle, _ptr(c), first, count, _ptr(mod_out),
                                            _stream(stream)))

    def rmsnorm_modulate(self, x, shift, scale, xm_out, stream=None) -> None:
        self._check(lib.h3dit_rmsnorm_modulate(self.handle, _ptr(x), _ptr(shift), _ptr(scale),
                                               _ptr(xm_out), x.shape[0], _stream(stream)))

    def rope_table(self, grids, n_txt: int, table_out, stream=None) -> None:
        g = grids_array(grids)
        self._check(lib.h3dit_rope_table(self.handle, g, len(grids), n_txt, _ptr(table_out),
                                         _stream(stream)))

    def linear(self, epilogue: int, a, w, out, gate=None, rope_table=None, stream=None) -> None:
        m, k = a.shape
        n = w.shape[0]
        self._check(lib.h3dit_linear(self.handle, epilogue, _ptr(a), _ptr(w), m, n, k, _ptr(out),
                                     _ptr(gate), _ptr(rope_table), _stream(stream)))

    def attention(self, q, k, v, ld_qkv: int, o, ld_o: int, n: int, stream=None) -> None:
        self._check(lib.h3dit_attention(self.handle, _ptr(q, False), _ptr(k, False),
                                        _ptr(v, False), ld_qkv, _ptr(o, False), ld_o, n,
                                        _stream(stream)))

    def empty(self, shape, kind: str):
        """A device buffer for the sequence-parallel driver: "act" and
        "exchange" (activations other ranks write into) are bf16; "fp8",
        "exchange_fp8" (E4M3 codes) and "sf", "exchange_sf" (MXFP8 scale
        bytes) are uint8; "f32" and "rope" are fp32."""
        import torch

        if kind in ("act", "exchange"):
            dt = torch.bfloat16
        elif kind in ("fp8", "exchange_fp8", "sf", "exchange_sf"):
            dt = torch.uint8
        else:
            dt = torch.float32
        return torch.empty(*shape, dtype=dt, device="cuda")

    def attention_heads(self, heads: int, q, k, v, ld_qkv: int, o, ld_o: int, n: int,
                        stream=None) -> None:
        self._check(lib.h3dit_attention_heads(self.handle, heads, _ptr(q, False), _ptr(k, False),
                                              _ptr(v, False), ld_qkv, _ptr(o, False), ld_o, n,
                                              _stream(stream)))

    def sp_pack_qkv(self, qkv, ranks: int, send, stream=None) -> None:
        """qkv [n_local, 3I] -> send [ranks][n_local][3I/ranks] (head groups)."""
        self._check(lib.h3dit_sp_pack_qkv(self.handle, _ptr(qkv), qkv.shape[0], ranks, _ptr(send),
                                          _stream(stream)))

    def sp_unpack_o(self, recv, ranks: int, o, stream=None) -> None:
        """recv [ranks][n_local][I/ranks] -> o [n_local, I]."""
        self._check(lib.h3dit_sp_unpack_o(self.handle, _ptr(recv), o.shape[0], ranks, _ptr(o),
                                          _stream(stream)))

    def sp_qkv_scatter(self, xm, w_qkv, rope_rows, recv_ptrs: Sequence[int], rank: int,
                       stream=None) -> None:
        """QKV + RoPE on this rank's rows xm [n_local, D], each head group's
        Q|K|V stored straight into rank g's receive buffer at device address
        recv_ptrs[g] (bf16 [ranks * n_local, 3I/ranks]): the first Ulysses
        all-to-all fused into the GEMM's epilogue."""
        arr = (C.c_void_p * len(recv_ptrs))(*recv_ptrs)
        self._check(lib.h3dit_sp_qkv_scatter(self.handle, _ptr(xm), xm.shape[0], _ptr(w_qkv),
                                             _ptr(rope_rows), arr, len(recv_ptrs), rank,
                                             _stream(stream)))

    def sp_attention_scatter(self, qkv_recv, o_ptrs: Sequence[int], rank: int,
                             stream=None) -> None:
        """Attention of this rank's head group over all tokens of qkv_recv
        [N, 3I/ranks], each output row stored straight into the out-projection
        input of the rank that holds it (device address o_ptrs[r], bf16
        [N / ranks, I]): the second all-to-all fused into the epilogue."""
        arr = (C.c_void_p * len(o_ptrs))(*o_ptrs)
        self._check(lib.h3dit_sp_attention_scatter(self.handle, _ptr(qkv_recv),
                                                   qkv_recv.shape[0], arr, len(o_ptrs), rank,
                                                   _stream(stream)))

    def sp_qkv_scatter_mx(self, xq, xq_sf, block: int, rope_rows, recv_ptrs: Sequence[int],
                          rank: int, stream=None) -> None:
        """sp_qkv_scatter for an MXFP8 context: this rank's quantized rows
        xq [n_local, D] (E4M3) with scales xq_sf, times the context's
        quantized QKV weights of `block`."""
        arr = (C.c_void_p * len(recv_ptrs))(*recv_ptrs)
        self._check(lib.h3dit_sp_qkv_scatter_mx(self.handle, _ptr(xq), _ptr(xq_sf), xq.shape[0],
                                                block, _ptr(rope_rows), arr, len(recv_ptrs), rank,
                                                _stream(stream)))

    def sp_attention_scatter_mx(self, qkv_recv, o_ptrs: Sequence[int], o_sf_ptrs: Sequence[int],
                                rank: int, stream=None) -> None:
        """sp_attention_scatter with MXFP8 output rows: E4M3 into o_ptrs[r]
        ([N / ranks, I]) and scales into o_sf_ptrs[r]."""
        if len(o_sf_ptrs) != len(o_ptrs):
            raise H3DitError(H3DIT_ERR_INVALID_ARG, "one scale array per output")
        arr = (C.c_void_p * len(o_ptrs))(*o_ptrs)
        sfa = (C.c_void_p * len(o_sf_ptrs))(*o_sf_ptrs)
        self._check(lib.h3dit_sp_attention_scatter_mx(self.handle, _ptr(qkv_recv),
                                                      qkv_recv.shape[0], arr, sfa, len(o_ptrs),
                                                      rank, _stream(stream)))

    def mx_scale_bytes(self, rows: int, k: int) -> int:
        return mx_scale_bytes(rows, k)

    def block_forward(self, block: int, t: float, x_img, grids, x_txt, mod=None,
                      stream=None) -> None:
        g = grids_array(grids)
        n_txt = 0 if x_txt is None else x_txt.shape[0]
        self._check(lib.h3dit_block_forward(self.handle, block, t, _ptr(mod), _ptr(x_img), g,
                                            len(grids), _ptr(x_txt), n_txt, _stream(stream)))

    def mx_quantize(self, src, dst, sf, stream=None) -> None:
        rows, k = src.shape
        self._check(lib.h3dit_mx_quantize(self.handle, _ptr(src), rows, k, _ptr(dst), _ptr(sf),
                                          _stream(stream)))

    def linear_mx(self, epilogue: int, a, a_sf, w, w_sf, out, out_sf=None, gate=None,
                  rope_table=None, stream=None) -> None:
        m, k = a.shape
        n = w.shape[0]
        self._check(lib.h3dit_linear_mx(self.handle, epilogue, _ptr(a), _ptr(a_sf), _ptr(w),
                                        _ptr(w_sf), m, n, k, _ptr(out), _ptr(out_sf), _ptr(gate),
                                        _ptr(rope_table), _stream(stream)))

    def block_linear_mx(self, block: int, which: int, a, a_sf, out, out_sf=None, gate=None,
                        rope_table=None, stream=None) -> None:
        self._check(lib.h3dit_block_linear_mx(self.handle, block, which, _ptr(a), _ptr(a_sf),
                                              a.shape[0], _ptr(out), _ptr(out_sf), _ptr(gate),
                                              _ptr(rope_table), _stream(stream)))

    def rmsnorm_modulate_mx(self, x, shift, scale, out, out_sf, stream=None) -> None:
        self._check(lib.h3dit_rmsnorm_modulate_mx(self.handle, _ptr(x), _ptr(shift), _ptr(scale),
                                                  _ptr(out), _ptr(out_sf), x.shape[0],
                                                  _stream(stream)))

    def attention_mx(self, q, k, v, ld_qkv: int, o, o_sf, n: int, stream=None) -> None:
        self._check(lib.h3dit_attention_mx(self.handle, _ptr(q, False), _ptr(k, False),
                                           _ptr(v, False), ld_qkv, _ptr(o), _ptr(o_sf), n,
                                           _stream(stream)))

    def embed_latent(self, latent, w_in, b_in, x_img_out, stream=None) -> None:
        """latent fp32 [C, Hl, Wl] -> x_img_out [(Hl/2)(Wl/2), D] in the token dtype."""
        ch, h, w = latent.shape
        self._check(lib.h3dit_embed_latent(self.handle, _ptr(latent), ch, h, w, _ptr(w_in),
                                           _ptr(b_in), _ptr(x_img_out), _stream(stream)))

    def output_modulation(self, c, w_mod, b_mod, mod_out, stream=None) -> None:
        self._check(lib.h3dit_output_modulation(self.handle, _ptr(c), _ptr(w_mod), _ptr(b_mod),
                                                _ptr(mod_out), _stream(stream)))

    def output_euler(self, x_img, mod, w_out, b_out, latent, dt: float, stream=None) -> None:
        """latent += dt * unpatchify(output layer(x_img)), in place."""
        ch, h, w = latent.shape
        self._check(lib.h3dit_output_euler(self.handle, _ptr(x_img), _ptr(mod), _ptr(w_out),
                                           _ptr(b_out), _ptr(latent), ch, h, w, dt,
                                           _stream(stream)))

    def denoise(self, io: dict, latent, x_txt, n_steps: int, stream=None) -> None:
        """latent fp32 [C, Hl, Wl]: noise in, the latent after n_steps Euler
        steps out; io holds w_in, b_in, w_mod, b_mod, w_out, b_out."""
        ch, h, w = latent.shape
        iw = h3dit_io_weights(_ptr(io["w_in"]), _ptr(io["b_in"]), _ptr(io["w_mod"]),
                              _ptr(io["b_mod"]), _ptr(io["w_out"]), _ptr(io["b_out"]))
        n_txt = 0 if x_txt is None else x_txt.shape[0]
        self._check(lib.h3dit_denoise(self.handle, C.byref(iw), _ptr(latent), ch, h, w,
                                      _ptr(x_txt), n_txt, n_steps, _stream(stream)))

    def selftest_bounded_wait(self, limit_us: int, stream=None) -> None:
        self._check(lib.h3dit_selftest_bounded_wait(self.handle, limit_us, _stream(stream)))

    def profile_begin(self) -> None:
        self._check(lib.h3dit_profile_begin(self.handle))

    def profile_end(self) -> dict:
        """{kind: (total ms, launches)} since profile_begin."""
        ms = (C.c_float * len(KERNEL_KINDS))()
        cnt = (C.c_int64 * len(KERNEL_KINDS))()
        self._check(lib.h3dit_profile_end(self.handle, ms, cnt))
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}

    def launch_count(self) -> int:
        return int(lib.h3dit_launch_count(self.handle))

    def step(self, t: float, x_img, grids, x_txt, stream=None) -> None:
        g = grids_array(grids)
        n_txt = 0 if x_txt is None else x_txt.shape[0]
        self._check(lib.h3dit_step(self.handle, t, _ptr(x_img), g, len(grids), _ptr(x_txt),
                                   n_txt, _stream(stream)))


def make_vae_config(width=1280, heads=10, head_dim=128, mlp=5120, layers=24, tile=32,
                    channels=24, max_tokens=65536, eps=1e-6) -> h3dit_vae_config:
    return h3dit_vae_config(width, heads, head_dim, mlp, layers, tile, channels, max_tokens, eps)


class VaeDecoder(Context):
    """A decoder context (h3dit_vae_create) holding the torch tensors it
    borrows. weights: w_in, b_in, lnf_g, lnf_b, w_out, b_out and "layers", a
    list of dicts with ln1_g, ln1_b, w_qkv, b_qkv, w_o, b_o, ln2_g, ln2_b, w_1,
    b_1, w_2, b_2 (matrices bf16, vectors fp32, all on the device)."""

    def __init__(self, cfg: h3dit_vae_config, weights: dict, stream=None, workspace=None):
        import torch

        self.cfg = cfg
        self._keep = [weights]
        ws_bytes = lib.h3dit_vae_workspace_bytes(C.byref(cfg))
        if ws_bytes == 0:
            raise H3DitError(H3DIT_ERR_INVALID_ARG, "invalid decoder config")
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        elif workspace.numel() * workspace.element_size() < ws_bytes:
            raise H3DitError(H3DIT_ERR_WORKSPACE, "workspace smaller than h3dit_vae_workspace_bytes")
        self.workspace = workspace
        names = [f[0] for f in h3dit_vae_layer_weights._fields_]
        layers = (h3dit_vae_layer_weights * len(weights["layers"]))()
        for i, lw in enumerate(weights["layers"]):
            layers[i] = h3dit_vae_layer_weights(*[_ptr(lw[k]) for k in names])
        self._layers = layers
        vw = h3dit_vae_weights(_ptr(weights["w_in"]), _ptr(weights["b_in"]), layers,
                               _ptr(weights["lnf_g"]), _ptr(weights["lnf_b"]),
                               _ptr(weights["w_out"]), _ptr(weights["b_out"]))
        handle = C.c_void_p()
        st = lib.h3dit_vae_create(C.byref(cfg), C.byref(vw), _ptr(workspace), ws_bytes,
                                  _stream(stream), C.byref(handle))
        check(None, st)
        self.handle = handle

    def decode(self, latent, image, stream=None) -> None:
        """latent fp32 [C, Hl, Wl] -> image fp32 [3, 16 Hl, 16 Wl]."""
        _, h, w = latent.shape
        self._check(lib.h3dit_vae_decode(self.handle, _ptr(latent), h, w, _ptr(image),
                                         _stream(stream)))
