"""Empty inputs through the C ABI: every stage entry point with a zero row or
token count succeeds without launching anything, for empty tensors (whose
device address is NULL), and leaves the context usable; negative counts and
bad shapes are still refused."""
import pytest

from image_generation_b200 import synth
from tests.helpers import block_tensors, time_tensors

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ctx(dims):
    from image_generation_b200 import h3dit as H

    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 1, 64)
    bw = block_tensors(synth.block_weights(dims, 0))
    return H.Context(cfg, time_tensors(synth.time_weights(dims, 0)), [bw]), bw


def _e(*shape, dt=None):
    return torch.empty(*shape, dtype=dt or torch.bfloat16, device="cuda")


def test_zero_row_calls_are_no_ops():
    from image_generation_b200 import h3dit as H

    d = synth.SMALL
    D, I, F, dh = d.hidden, d.inner, d.ffn, d.head_dim
    ctx, bw = _ctx(d)
    f32 = torch.float32
    x0, xm0, sh = _e(0, D, dt=f32), _e(0, D), torch.zeros(D, device="cuda")
    q = _e(0, 3 * I)
    n0 = ctx.launch_count()
    ctx.rmsnorm_modulate(x0, sh, sh, xm0)
    ctx.layernorm(x0, sh, sh, xm0)
    for epi, out in ((H.H3DIT_EPI_STORE, _e(0, F)), (H.H3DIT_EPI_GELU, _e(0, F))):
        ctx.linear(epi, xm0, bw["w_ff1"], out)
    ctx.linear(H.H3DIT_EPI_GATED_RESIDUAL, _e(0, F), bw["w_ff2"], x0, gate=sh)
    ctx.linear(H.H3DIT_EPI_QKV_ROPE, xm0, bw["w_qkv"], q, rope_table=_e(0, dh // 2, 2, dt=f32))
    ctx.linear_bias(H.H3DIT_EPI_STORE, xm0, bw["w_ff1"], torch.zeros(F, device="cuda"), _e(0, F))
    ctx.attention(q[:, :I], q[:, I:2 * I], q[:, 2 * I:], 3 * I, _e(0, I), I, 0)
    ctx.attention_heads(2, q[:, :I], q[:, I:2 * I], q[:, 2 * I:], 3 * I, _e(0, I), I, 0)
    ctx.attention_batched(q[:, :I], q[:, I:2 * I], q[:, 2 * I:], 3 * I, _e(0, I), I, 0, 3)
    ctx.sp_pack_qkv(q, 2, _e(2, 0, 3 * I // 2))
    ctx.sp_unpack_o(_e(2, 0, I // 2), 2, _e(0, I))
    ctx.sp_qkv_scatter(xm0, bw["w_qkv"], _e(0, dh // 2, 2, dt=f32), [0, 0], 1)
    ctx.sp_attention_scatter(_e(0, 3 * I // 2), [0, 0], 0)
    ctx.rope_table([], 0, _e(0, dh // 2, 2, dt=f32))
    ctx.mx_quantize(_e(0, D), _e(0, D, dt=torch.uint8), _e(0, dt=torch.uint8))
    assert ctx.launch_count() == n0
    assert ctx.sync_status() == 0


def test_counts_and_shapes_are_still_checked_with_no_rows():
    from image_generation_b200 import h3dit as H

    d = synth.SMALL
    ctx, bw = _ctx(d)
    bad = [
        # a weight whose K is not a multiple of the 64-deep k-block
        (lambda: ctx.linear(H.H3DIT_EPI_STORE, _e(0, 100), _e(32, 100), _e(0, 32)),
         H.H3DIT_ERR_UNSUPPORTED),
        # more heads than the context has, with no tokens
        (lambda: ctx.attention_heads(9, _e(0, 768), _e(0, 768), _e(0, 768), 3 * 768, _e(0, 768),
                                     768, 0), H.H3DIT_ERR_INVALID_ARG),
        # ranks that do not divide the heads, with no tokens
        (lambda: ctx.sp_pack_qkv(_e(0, 3 * d.inner), 3, _e(3, 0, d.inner)),
         H.H3DIT_ERR_UNSUPPORTED),
        # a rank outside [0, ranks), with no tokens
        (lambda: ctx.sp_attention_scatter(_e(0, 3 * d.inner // 2), [0, 0], 2),
         H.H3DIT_ERR_INVALID_ARG),
    ]
    for call, status in bad:
        with pytest.raises(H.H3DitError) as e:
            call()
        assert e.value.status == status
    assert ctx.sync_status() == 0
