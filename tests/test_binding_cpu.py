"""Argument checks of the Python binding (no GPU).

The C ABI takes plain pointers and sizes, so the binding checks every
tensor's shape and dtype against the sizes it passes, before any call: a
tensor smaller than its sizes say would otherwise be read or written out of
bounds.  Device-only entry points also refuse host tensors."""

import pytest
import torch

import differential_attention_transformers_b200 as da

bf, f32 = torch.bfloat16, torch.float32


def z(*shape, dtype=bf):
    return torch.zeros(*shape, dtype=dtype)


def test_prefill_shapes():
    q, k, v, lam = z(1, 4, 16, 128), z(1, 2, 32, 128), z(1, 2, 32, 128), z(2, dtype=f32)
    with pytest.raises(ValueError, match="v has shape"):
        da.fwd_v2(q, k, z(1, 2, 31, 128), lam)
    with pytest.raises(ValueError, match="lam has shape"):
        da.fwd_v2(q, k, v, z(3, dtype=f32))
    with pytest.raises(ValueError, match="lam must be"):
        da.fwd_v2(q, k, v, z(2, dtype=torch.float64))
    with pytest.raises(ValueError, match="k must be"):
        da.fwd_v2(q, k.float(), v, lam)
    with pytest.raises(ValueError, match="out has shape"):
        da.fwd_v2(q, k, v, lam, out=z(1, 2, 15, 128))
    with pytest.raises(ValueError, match="4-d"):
        da.fwd_v2(z(4, 16, 128), k, v, lam)
    q1, k1, vv = z(2, 4, 16, 64), z(2, 2, 32, 64), z(2, 2, 32, 128)
    with pytest.raises(ValueError, match="k2 has shape"):
        da.fwd_v1(q1, k1, q1, z(2, 2, 32, 32), vv, z(4, dtype=f32))
    with pytest.raises(ValueError, match="q2 has shape"):
        da.fwd_v1(q1, k1, z(2, 4, 17, 64), k1, vv, z(4, dtype=f32))


def test_decode_shapes():
    q, kc = z(2, 8, 128), z(2, 2, 100, 128)
    with pytest.raises(ValueError, match="vc has shape"):
        da.decode_v2(q, kc, z(2, 2, 99, 128), z(4, dtype=f32))
    with pytest.raises(ValueError, match="3-d"):
        da.decode_v2(z(2, 8, 1, 128), kc, kc, z(4, dtype=f32))
    q1, k1, v = z(2, 4, 64), z(2, 1, 50, 64), z(2, 1, 50, 128)
    with pytest.raises(ValueError, match="v has shape"):
        da.decode_v1(q1, k1, q1, k1, z(3, 1, 50, 128), z(4, dtype=f32))
    with pytest.raises(ValueError, match="out has shape"):
        da.decode_v1(q1, k1, q1, k1, v, z(4, dtype=f32), out=z(2, 4, 64))
    kp = z(10, 16, 2, 128)
    bt, sl = z(2, 4, dtype=torch.int32), z(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="v_pages has shape"):
        da.decode_v2_paged(q, kp, z(10, 16, 1, 128), bt, sl, z(4, dtype=f32))
    with pytest.raises(ValueError, match="block_table must be"):
        da.decode_v2_paged(q, kp, kp, bt.long(), sl, z(4, dtype=f32))
    with pytest.raises(ValueError, match="seq_lens has shape"):
        da.decode_v2_paged(q, kp, kp, bt, z(3, dtype=torch.int32), z(4, dtype=f32))


def test_training_shapes_and_device():
    q, k, lam = z(1, 4, 16, 128), z(1, 2, 16, 128), z(2, dtype=f32)
    lse, om, dout = z(1, 2, 2, 16, dtype=f32), z(1, 2, 2, 16, 128), z(1, 2, 16, 128)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        da.fwd_v2_train(q, k, k, lam)
    with pytest.raises(ValueError, match="q must be"):
        da.fwd_v2_train(q.float(), k, k, lam)
    with pytest.raises(ValueError, match="lse has shape"):
        da.bwd_v2(q, k, k, lam, dout, z(1, 2, 16, dtype=f32), om)
    with pytest.raises(ValueError, match="o_maps has shape"):
        da.bwd_v2(q, k, k, lam, dout, lse, z(1, 2, 16, 128))
    with pytest.raises(ValueError, match="dout has shape"):
        da.bwd_v2(q, k, k, lam, z(1, 4, 16, 128), lse, om)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        da.bwd_v2(q, k, k, lam, dout, lse, om)
    q1, k1, v = z(1, 2, 16, 64), z(1, 1, 16, 64), z(1, 1, 16, 128)
    lam1, lse1, om1, d1 = z(2, dtype=f32), z(1, 2, 2, 16, dtype=f32), z(1, 2, 2, 16, 128), z(1, 2, 16, 128)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        da.fwd_v1_train(q1, k1, q1, k1, v, lam1, rmsnorm=True)
    with pytest.raises(ValueError, match="rstd is required"):
        da.bwd_v1(q1, k1, q1, k1, v, lam1, d1, d1, lse1, om1, None, rmsnorm=True)
    with pytest.raises(ValueError, match="out has shape"):
        da.bwd_v1(q1, k1, q1, k1, v, lam1, d1, z(1, 2, 15, 128), lse1, om1, z(1, 2, 16, dtype=f32),
                  z(1, 2, 16, dtype=f32), rmsnorm=True)
    with pytest.raises(ValueError, match="o2c is required"):
        da.bwd_v1(q1, k1, q1, k1, v, lam1, d1, d1, lse1, om1, z(1, 2, 16, dtype=f32), None, rmsnorm=True)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        da.bwd_v1(q1, k1, q1, k1, v, lam1, d1, None, lse1, om1, None, rmsnorm=False)
    p = [z(3, 8, dtype=f32) for _ in range(4)]
    with pytest.raises(ValueError, match="dlam has shape"):
        da.lambda_backward(*p, z(4, dtype=f32))
    with pytest.raises(ValueError, match="lk2 has shape"):
        da.lambda_backward(p[0], p[1], p[2], z(3, 7, dtype=f32), z(3, dtype=f32))


def test_lowrank_shapes_and_device():
    q, k, lam = z(1, 4, 16, 128), z(1, 2, 20, 128), z(4, dtype=f32)
    F, G = z(4, 16, 3, dtype=f32), z(4, 20, 3, dtype=f32)
    with pytest.raises(ValueError, match="G has shape"):
        da.fwd_lowrank(q, k, k, F, z(4, 19, 3, dtype=f32), lam)
    with pytest.raises(ValueError, match="F has shape"):
        da.fwd_lowrank(q, k, k, z(4, 15, 3, dtype=f32), G, lam)
    with pytest.raises(ValueError, match="lam has shape"):
        da.fwd_lowrank(q, k, k, F, G, z(2, dtype=f32))
    with pytest.raises(ValueError, match="v must be"):
        da.fwd_lowrank(q, k, k.float(), F, G, lam)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        da.fwd_lowrank(q, k, k, F, G, lam)
