"""The Python binding checks every tensor against the layouts of include/mala.h before it
hands pointers to the C ABI (shapes, dtypes, contiguity, one device), and only then asks
for a CUDA device.  These tests run on CPU tensors: a well-formed call must get as far as
the device check, and each malformed argument must be named in the error."""

import numpy as np
import pytest
import torch


@pytest.fixture(scope="module")
def mala():
    from mass_adaptive_sparse_fwd_b200 import build

    build.build_library()
    from mass_adaptive_sparse_fwd_b200 import mala

    return mala


bf = torch.bfloat16
f32 = torch.float32


def _train(B=1, L=300, H=4, Hkv=2, d=64, dt=bf):
    Q = torch.zeros(B, L, H, d, dtype=dt)
    K = torch.zeros(B, L, Hkv, d, dtype=dt)
    V = torch.zeros(B, L, Hkv, d, dtype=dt)
    return Q, K, V


def _reaches_device_check(call):
    with pytest.raises(ValueError, match="CUDA device"):
        call()


def test_well_formed_calls_reach_the_device_check(mala):
    B, L, H, Hkv, d = 2, 300, 4, 2, 64
    T = mala.n_tiles(L)
    Q, K, V = _train(B, L, H, Hkv, d)
    O, LSE = torch.zeros_like(Q), torch.zeros(B, H, L)
    mask = torch.zeros(B, H, T, T, dtype=torch.uint8)
    ws = torch.zeros(4096, dtype=torch.uint8)
    _reaches_device_check(lambda: mala.mala_fwd(Q, K, V, 0.1, 1.0))
    _reaches_device_check(lambda: mala.mala_fwd(Q, K, V, 0.1, 1.0, O=O, LSE=LSE, workspace=ws,
                                                tile_mask=mask))
    _reaches_device_check(lambda: mala.mala_bwd(Q, K, V, O, LSE, Q, 0.1, 1.0, tile_mask=mask))
    # fp32 path
    Qf, Kf, Vf = _train(B, L, H, Hkv, d, f32)
    _reaches_device_check(lambda: mala.mala_fwd(Qf, Kf, Vf, 0.1, 1.0))
    # prefill: 100 queries at the end of 300 keys
    Qc = torch.zeros(B, 100, H, d, dtype=bf)
    pm = torch.zeros(B, H, 1, T, dtype=torch.uint8)
    _reaches_device_check(lambda: mala.mala_fwd_prefill(Qc, K, V, 0.1, 1.0, tile_mask=pm))
    # packed batch
    cu_q, cu_k = [0, 100, 130], [0, 200, 230]
    _reaches_device_check(lambda: mala.mala_fwd_varlen(
        torch.zeros(130, H, d, dtype=bf), torch.zeros(230, Hkv, d, dtype=bf),
        torch.zeros(230, Hkv, d, dtype=bf), cu_q, cu_k, 0.1, 1.0))
    # decode
    q = torch.zeros(B, H, d, dtype=bf)
    dm = torch.zeros(B, H, T, dtype=torch.uint8)
    _reaches_device_check(lambda: mala.mala_decode(q, K, V, 0.1, 1.0, tile_mask=dm))
    _reaches_device_check(lambda: mala.mala_decode_noalloc(q, K, V, 0.1, 1.0))


@pytest.mark.parametrize("case", [
    "K_rows", "V_heads", "K_dtype", "O_shape", "LSE_dtype", "LSE_shape", "Q_noncontig",
    "mask_small", "mask_dtype", "Q_dtype"])
def test_forward_rejects_malformed_tensors(mala, case):
    B, L, H, Hkv, d = 1, 300, 4, 2, 64
    Q, K, V = _train(B, L, H, Hkv, d)
    kw = {}
    if case == "K_rows":
        K = torch.zeros(B, L - 1, Hkv, d, dtype=bf)
    elif case == "V_heads":
        V = torch.zeros(B, L, Hkv + 1, d, dtype=bf)
    elif case == "K_dtype":
        K = K.float()
    elif case == "O_shape":
        kw["O"] = torch.zeros(B, L, H, d + 1, dtype=bf)
    elif case == "LSE_dtype":
        kw["LSE"] = torch.zeros(B, H, L, dtype=bf)
    elif case == "LSE_shape":
        kw["LSE"] = torch.zeros(B, L, H)
    elif case == "Q_noncontig":
        Q = torch.zeros(B, H, L, d, dtype=bf).transpose(1, 2)
    elif case == "mask_small":
        kw["tile_mask"] = torch.zeros(B * H * 3 * 3 - 1, dtype=torch.uint8)
    elif case == "mask_dtype":
        kw["tile_mask"] = torch.zeros(B, H, 3, 3, dtype=torch.int32)
    elif case == "Q_dtype":
        Q = Q.half()
    with pytest.raises((TypeError, ValueError)) as e:
        mala.mala_fwd(Q, K, V, 0.1, 1.0, **kw)
    assert "CUDA device" not in str(e.value)
    named = {"K_rows": "K", "V_heads": "V", "K_dtype": "K", "O_shape": "O", "LSE_dtype": "LSE",
             "LSE_shape": "LSE", "Q_noncontig": "Q", "mask_small": "tile_mask",
             "mask_dtype": "tile_mask", "Q_dtype": "dtype"}[case]
    assert named in str(e.value)


def test_backward_and_decode_reject_malformed_tensors(mala):
    B, L, H, Hkv, d = 1, 300, 4, 2, 64
    Q, K, V = _train(B, L, H, Hkv, d)
    O, LSE = torch.zeros_like(Q), torch.zeros(B, H, L)
    with pytest.raises(ValueError, match="dO"):
        mala.mala_bwd(Q, K, V, O, LSE, torch.zeros(B, L, H, d + 2, dtype=bf), 0.1, 1.0)
    with pytest.raises(ValueError, match="dK"):
        mala.mala_bwd(Q, K, V, O, LSE, Q, 0.1, 1.0, dK=torch.zeros_like(Q))
    q = torch.zeros(B, H, d, dtype=bf)
    with pytest.raises(ValueError, match="Vc"):
        mala.mala_decode(q, K, torch.zeros(B, L + 1, Hkv, d, dtype=bf), 0.1, 1.0)
    with pytest.raises(ValueError, match="Kc"):
        mala.mala_decode_noalloc(q, torch.zeros(B, L, Hkv, d + 1, dtype=bf), V, 0.1, 1.0)
    with pytest.raises(ValueError, match="tile_mask"):
        mala.mala_decode(q, K, V, 0.1, 1.0, tile_mask=torch.zeros(B * H * 2, dtype=torch.uint8))
    with pytest.raises(ValueError, match="LSE"):
        mala.mala_decode(q, K, V, 0.1, 1.0, LSE=torch.zeros(B, H + 1))


def test_packed_batch_offsets_must_match_the_tensors(mala):
    H, Hkv, d = 4, 2, 64
    Q = torch.zeros(130, H, d, dtype=bf)
    K = torch.zeros(230, Hkv, d, dtype=bf)
    with pytest.raises(ValueError, match="cu_seqlens_q"):
        mala.mala_fwd_varlen(Q, K, K, [0, 100, 131], [0, 200, 230], 0.1, 1.0)
    with pytest.raises(ValueError, match="K"):
        mala.mala_fwd_varlen(Q, K, K, [0, 100, 130], [0, 200, 231], 0.1, 1.0)
    with pytest.raises(ValueError, match="offsets"):
        mala.mala_fwd_varlen(Q, K, K, [0, 100, 130], [0, 230], 0.1, 1.0)
    with pytest.raises(ValueError, match="offsets"):
        mala.mala_fwd_varlen(Q, K, K, np.array([130]), np.array([230]), 0.1, 1.0)


def test_workspace_size_counts_bytes(mala):
    ws = torch.zeros(10, dtype=torch.float32)
    assert mala._workspace_bytes("t", ws, ws.device) == 40
    assert mala._workspace_bytes("t", None, ws.device) == 0
    with pytest.raises(ValueError, match="workspace"):
        mala._workspace_bytes("t", torch.zeros(4, 4)[:, 0], ws.device)
