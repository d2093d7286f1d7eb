"""The C-ABI library loads on a machine without a GPU, exports every entry point that
include/dust.h declares, and rejects bad arguments before touching the device (CPU only)."""
import ctypes
import os
import re

import pytest

import zeroth_order_transformer_b200 as z

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(dust_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    lib = z.lib()
    decl = declared_functions()
    assert {"dust_noisy_linear_fwd", "dust_credit", "dust_weight_grad"} <= decl
    for name in decl:
        assert hasattr(lib, name), name
    assert set(z.EXPORTED_SYMBOLS) <= decl


def test_status_strings():
    for code, name in [(0, "DUST_OK"), (1, "DUST_ERR_INVALID_ARG"), (2, "DUST_ERR_UNSUPPORTED"),
                       (3, "DUST_ERR_CUDA"), (4, "DUST_ERR_TIMEOUT"), (5, "DUST_ERR_WORKSPACE")]:
        assert z.status_string(code) == name


def test_workspace_sizes_are_positive_and_grow():
    a = z.dust_workspace_size(z.DUST_OP_NOISY_LINEAR_FWD, z.DUST_BF16, 8192, 768, 3072, 16)
    b = z.dust_workspace_size(z.DUST_OP_NOISY_LINEAR_FWD, z.DUST_BF16, 8192, 768, 3072, 32)
    assert 0 < a < b
    assert z.dust_workspace_size(z.DUST_OP_CREDIT, z.DUST_F32, 32768, 0, 0, 32) > 0
    assert z.dust_workspace_size(z.DUST_OP_WEIGHT_GRAD, z.DUST_BF16, 8192, 768, 3072, 16) >= 8192 * 3072 * 2


def _fwd(**kw):
    args = dict(x=0x1000, W=0x1000, u=0x1000, dt=z.DUST_BF16, N=256, d_in=64, d_out=64, K=4,
                sigma=1e-3, key=z.NoiseKey(1).c(), dloss=0x1000, ld=256, ws=None, nb=0, s=None)
    args.update(kw)
    return z.lib().dust_noisy_linear_fwd(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), z.DUST_ERR_INVALID_ARG),
    (dict(x=None), z.DUST_ERR_INVALID_ARG),
    (dict(x=0x1008), z.DUST_ERR_INVALID_ARG),            # misaligned
    (dict(K=0), z.DUST_ERR_INVALID_ARG),
    (dict(ld=100), z.DUST_ERR_INVALID_ARG),
    (dict(d_out=72), z.DUST_ERR_UNSUPPORTED),            # bf16 needs multiples of 16
    (dict(dt=7), z.DUST_ERR_INVALID_ARG),
    (dict(sigma=float("nan")), z.DUST_ERR_INVALID_ARG),
    (dict(ws=None, nb=0), z.DUST_ERR_WORKSPACE),
])
def test_fwd_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


def test_credit_and_weight_grad_reject_bad_arguments():
    L = z.lib()
    # K < 2: the centred loss is identically zero
    assert L.dust_credit(0x1000, 256, 1, 256, 0x1000, 1, 0.9, 0x1000, 256, None, 0, None) == 1
    assert L.dust_credit(0x1000, 256, 4, 256, 0x1000, 1, 1.5, 0x1000, 256, None, 0, None) == 1
    assert L.dust_credit(0x1000, 256, 4, 256, 0x1000, 1, 0.9, 0x1000, 256, None, 0, None) == 5
    key = z.NoiseKey(1).c()
    # sigma must be > 0 (division by sigma); K_total >= K_chunk
    assert L.dust_weight_grad(0x1000, 256, 0x1000, 1, 256, 64, 64, 4, 4, 0.0, key, 0x1000, 0,
                              None, 2, None, 0, None) == 1
    assert L.dust_weight_grad(0x1000, 256, 0x1000, 1, 256, 64, 64, 4, 2, 1e-3, key, 0x1000, 0,
                              None, 2, None, 0, None) == 1
    bad = z.dust_noise_key(1, 0, 0xFFFFFFFF, 0, 0)   # draw index would wrap
    assert L.dust_weight_grad(0x1000, 256, 0x1000, 1, 256, 64, 64, 4, 4, 1e-3, bad, 0x1000, 0,
                              None, 2, None, 0, None) == 1
    # g enters the contraction as one or two bf16 terms, nothing else
    for terms in (0, 3, -1):
        assert L.dust_weight_grad(0x1000, 256, 0x1000, 1, 256, 64, 64, 4, 4, 1e-3, key, 0x1000,
                                  0, None, terms, None, 0, None) == 1


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "zeroth_order_transformer_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "dust_oracle" not in src, fn


def test_forward_plan():
    """The bf16 forward's form and tail split (host logic, 148 SMs: 296 CTA slots of the
    one-tile kernel)."""
    sms = 148
    # 8 x 1024 tokens, 768 -> 3072: 768 tiles, under three waves of 296: persistent
    assert z.dust_debug_fwd_plan(8192, 16, [3072], sms) == (True, 0)
    assert z.dust_debug_fwd_plan(1024, 16, [3072], sms) == (True, 0)
    assert z.dust_debug_fwd_plan(128, 4, [256], sms) == (True, 0)
    # 887 tiles persistent, 888 (three waves) one tile per CTA
    assert z.dust_debug_fwd_plan(887 * 128, 8, [256], sms)[0]
    assert not z.dust_debug_fwd_plan(888 * 128, 8, [256], sms)[0]
    # 32k tokens x 1024 -> 1024, K = 32: 1024 tiles; the 136 of the last wave in two ranges
    # of 32 units (eight rounds of the four warp groups: one wave of 272 CTAs)
    assert z.dust_debug_fwd_plan(32768, 32, [1024], sms) == (False, 2)
    # 16k x 2048 -> 8192, K = 64: 4096 tiles, 248 in the last wave, whole
    assert z.dust_debug_fwd_plan(16384, 64, [8192], sms) == (False, 1)
    # the 48-layer group: 20736 tiles
    assert not z.dust_debug_fwd_plan(8192, 16, [2304, 768, 3072, 768] * 12, sms)[0]
    rng = __import__("random").Random(3)
    for _ in range(200):
        N, K = rng.randrange(1, 200000), rng.randrange(1, 70)
        d = [16 * rng.randrange(1, 600) for _ in range(rng.randrange(1, 5))]
        persistent, split = z.dust_debug_fwd_plan(N, K, d, sms)
        tiles = sum(-(-N // 128) * -(-dd // 256) for dd in d)
        assert persistent == (tiles < 3 * 2 * sms)
        assert (split == 0) if persistent else (1 <= split <= 8 and (2 * K) // split >= 1)


@pytest.mark.parametrize("args", [
    (0, 4, [256], 148), (128, 0, [256], 148), (128, 4, [0], 148), (128, 4, [256], 0),
])
def test_forward_plan_rejects_bad_arguments(args):
    with pytest.raises(z.DustError):
        z.dust_debug_fwd_plan(*args)
