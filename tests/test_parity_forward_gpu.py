"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small and shrunken cases are compared on every element; the full-size
workloads on a seeded sample of rows (edges included) that the oracle
computes one by one.  Tolerances: fp32 max abs 1e-4; bf16 max abs 2e-2 and
mean abs 2e-3; lse abs 1e-3.  Every output lives inside NaN guard bands that
must survive the launch.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, F32_MAX_ABS, LSE_ABS, check_guards, compare,
                      guarded, sample_rows)
from sliding_window_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


def run_forward(swa, q, k, v, L, R, d=1, bs=0, G=None, scale=0.0, f32=False):
    B, N, H, D = q.shape
    dt = torch.float32 if f32 else torch.bfloat16
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    obuf, out = guarded((B, N, H, D), dt)
    lbuf, lse = guarded((B, H, N), torch.float32)
    Gd = None if G is None or len(G) == 0 else torch.as_tensor(G, dtype=torch.int32).cuda()
    if f32:
        swa.swa_forward_f32(qd, kd, vd, out, lse, L, R, d, bs, Gd, scale)
    elif bs:
        swa.swa_forward_ex(qd, kd, vd, out, lse, L, R, d, bs, Gd, scale)
    else:
        swa.swa_forward(qd, kd, vd, out, lse, L, R, d, Gd, scale)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    check_guards(obuf)
    check_guards(lbuf)
    return out.float().cpu().numpy(), lse.cpu().numpy()


def full_check(swa, cfg_or_args, f32=False):
    q, k, v, L, R, d, bs, G, scale = cfg_or_args
    out, lse = run_forward(swa, q, k, v, L, R, d, bs, G, scale, f32)
    ref_o, ref_l = oracle.forward(q, k, v, L, R, d, bs, [] if G is None else G, scale)
    if f32:
        compare(out, ref_o, F32_MAX_ABS, what="out")
        compare(lse, ref_l, F32_MAX_ABS, what="lse")
    else:
        compare(out, ref_o, BF16_MAX_ABS, BF16_MEAN_ABS, what="out")
        compare(lse, ref_l, LSE_ABS, what="lse")


def rand_case(B, N, H, Hkv, D, seed, dtype=torch.bfloat16):
    q = inputs.normal((B, N, H, D), seed, 0, dtype)
    k = inputs.normal((B, N, Hkv, D), seed, 1, dtype)
    v = inputs.normal((B, N, Hkv, D), seed, 2, dtype)
    return q, k, v


# ------------------------------------------------------------------ fp32 path
def test_config_tiny_bidirectional_fp32(swa):
    cfg = inputs.CONFIGS["tiny_bidir_fp32"]
    q, k, v, G = inputs.forward_inputs(cfg)
    full_check(swa, (q, k, v, cfg.win_left, cfg.win_right, 1, 0, None, cfg.scale), f32=True)


@pytest.mark.parametrize("case", [
    # (B, N, H, Hkv, D, L, R, d, bs, G)
    (1, 100, 4, 2, 64, 10, 0, 1, 0, None),
    (2, 77, 2, 1, 32, 5, 5, 3, 0, None),
    (1, 130, 2, 2, 96, 64, 64, 2, 16, None),
    (1, 90, 2, 2, 128, 4, 4, 1, 0, [0, 30, 89]),
    (1, 90, 2, 2, 64, 6, 0, 1, 0, [0, 45]),
    (1, 1, 1, 1, 64, 3, 3, 1, 0, None),
    (1, 50, 2, 1, 64, -1, -1, 1, 0, None),
])
def test_fp32_variants(swa, case):
    B, N, H, Hkv, D, L, R, d, bs, G = case
    q, k, v = rand_case(B, N, H, Hkv, D, 31, torch.float32)
    full_check(swa, (q, k, v, L, R, d, bs, G, 0.0), f32=True)


# ------------------------------------------------------------ bf16 tcgen05 path
SMALL_BF16 = [
    # (B, N, H, Hkv, D, L, R, d, bs, G)
    (1, 128, 1, 1, 128, 127, 0, 1, 0, None),       # one full causal tile
    (1, 256, 2, 1, 128, 300, 0, 1, 0, None),       # window longer than N
    (1, 1000, 8, 2, 128, 300, 0, 1, 0, None),      # ragged tail, GQA 4
    (1, 129, 2, 2, 64, 64, 64, 1, 0, None),        # tile + 1
    (1, 127, 2, 2, 64, 16, 16, 1, 0, None),        # tile - 1
    (1, 1, 1, 1, 128, 5, 0, 1, 0, None),           # N = 1
    (2, 300, 2, 2, 64, 0, 0, 1, 0, None),          # one-key window
    (1, 400, 2, 1, 128, -1, -1, 1, 0, None),       # unbounded = full attention
    (1, 500, 2, 2, 64, -1, 0, 1, 0, None),         # unbounded causal
    (2, 700, 3, 3, 64, 40, 40, 1, 0, [0, 128, 256, 384, 512, 640]),
    (1, 600, 4, 2, 128, 100, 0, 1, 0, [0, 7, 300]),  # causal + globals
    (1, 1003, 2, 2, 64, 50, 50, 3, 0, None),       # dilated, N mod d != 0
    (1, 2000, 2, 2, 128, 20, 30, 16, 0, None),     # d > 8 classes per launch
    (1, 1344, 2, 1, 64, 128, 128, 4, 64, None),    # block-level dilation
    (1, 1000, 2, 2, 64, 128, 0, 2, 64, [3, 500]),  # block, causal, ragged, globals
    (1, 500, 8, 1, 128, 64, 64, 1, 0, [0, 250]),   # globals with a GQA group of 8
    (1, 400, 8, 2, 64, 40, 0, 1, 0, [5, 399]),     # globals, GQA 4, causal, last row global
    # global query rows run inside the fused launch (global tiles of up to
    # 128 rows each, every key of the sequence):
    (1, 300, 32, 2, 128, 30, 30, 1, 0, [0, 100, 299]),        # GQA 16 with globals
    (1, 700, 4, 4, 64, 20, 0, 1, 0, list(range(0, 700, 4))),  # 175 globals: two global tiles
    (2, 900, 2, 2, 64, 16, 16, 4, 0, [1, 2, 450, 899]),       # token dilation + globals
    (1, 96, 2, 1, 128, 3, 3, 1, 0, list(range(96))),          # every row global = full attention
    (1, 260, 3, 3, 128, 10, 0, 1, 0, [129, 130, 259]),        # odd head count, causal
    # query tiles whose rows take no global key skip the global-key tiles:
    # causal sinks inside the first tiles' bands, and globals inside the
    # band on both sides of a bidirectional window
    (1, 1200, 4, 2, 128, 300, 0, 1, 0, [0, 1, 2, 3]),          # sinks: tiles 0-2 skip
    (1, 1100, 4, 4, 64, 300, 0, 1, 0, [0, 2, 130, 131]),        # sinks + a later global
    (1, 900, 2, 2, 128, 400, 400, 1, 0, [300, 350]),            # in every band of tiles 0-4
]


@pytest.mark.parametrize("case", SMALL_BF16)
def test_bf16_small(swa, case):
    B, N, H, Hkv, D, L, R, d, bs, G = case
    q, k, v = rand_case(B, N, H, Hkv, D, 7)
    full_check(swa, (q, k, v, L, R, d, bs, G, 0.0))


@pytest.mark.parametrize("name", ["small_causal", "small_global", "small_dilated", "small_block"])
def test_bf16_shrunken_configs(swa, name):
    cfg = inputs.CONFIGS[name]
    q, k, v, G = inputs.forward_inputs(cfg)
    full_check(swa, (q, k, v, cfg.win_left, cfg.win_right, cfg.dilation, cfg.dilation_block,
                     G.numpy() if len(G) else None, cfg.scale))


def test_bf16_large_scores_rescale(swa):
    """Scores that grow along the row force the lazy max rescaling path."""
    B, N, H, D = 1, 1024, 2, 128
    q, k, v = rand_case(B, N, H, H, D, 11)
    ramp = torch.linspace(0.1, 4.0, N).view(1, N, 1, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float() * 2.0).to(torch.bfloat16)
    full_check(swa, (q, k, v, 900, 0, 1, 0, None, 0.0))


# ------------------------------------------------------- full-size workloads
@pytest.mark.parametrize("name", ["mistral_causal_prefill", "longformer_global", "dilated_token",
                                  "dilated_block"])
def test_full_size_sampled(swa, name):
    cfg = inputs.CONFIGS[name]
    q, k, v, G = inputs.forward_inputs(cfg)
    Gn = G.numpy() if len(G) else None
    out, lse = run_forward(swa, q, k, v, cfg.win_left, cfg.win_right, cfg.dilation,
                           cfg.dilation_block, Gn, cfg.scale)
    N = cfg.N
    edges = [0, 1, 127, 128, 129, 511, 512, 513, 4095, 4096, N // 2, N - 129, N - 128, N - 2,
             N - 1]
    rows = sample_rows(cfg.B, cfg.H, N, 1500, seed=5, extra_i=edges)
    ref_o, ref_l = oracle.forward(q, k, v, cfg.win_left, cfg.win_right, cfg.dilation,
                                  cfg.dilation_block, [] if Gn is None else Gn, cfg.scale,
                                  rows=rows)
    got_o = out[rows[:, 0], rows[:, 2], rows[:, 1]]
    got_l = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    compare(got_o, ref_o, BF16_MAX_ABS, BF16_MEAN_ABS, what=f"{name} out")
    compare(got_l, ref_l, LSE_ABS, what=f"{name} lse")
    assert np.isfinite(out).all()


@pytest.mark.parametrize("D,H,Hkv", [(128, 4, 2), (64, 2, 2), (128, 3, 3)])
def test_bf16_score_jumps(swa, D, H, Hkv):
    """A few keys with huge scores appear late in a row's window: the running
    max jumps by far more than 2^64 in both halves of a key tile, which forces
    the kernel to rescale O, l and the already written P."""
    B, N = 1, 1024
    q, k, v = rand_case(B, N, H, Hkv, D, 23)
    k = k.float()
    for pos in (300, 330, 700, 770, 1000):  # first and second halves of key tiles
        k[:, pos] *= 40.0
    k = k.to(torch.bfloat16)
    full_check(swa, (q, k, v, 600, 0, 1, 0, None, 0.0))
    full_check(swa, (q, k, v, 200, 200, 1, 0, None, 0.0))


def test_globals_allocate_nothing(swa):
    """The forward with global tokens runs in one launch with no library
    workspace: after swa_release() the device's free memory is unchanged by
    the call (torch's own tensors are made before the first reading)."""
    cfg = inputs.CONFIGS["small_global"]
    q, k, v, G = inputs.forward_inputs(cfg)
    qd, kd, vd, Gd = q.cuda(), k.cuda(), v.cuda(), G.cuda()
    out = torch.empty_like(qd)
    lse = torch.empty(cfg.B, cfg.H, cfg.N, device="cuda")
    swa.swa_release()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    swa.swa_forward(qd, kd, vd, out, lse, cfg.win_left, cfg.win_right, cfg.dilation, Gd,
                    cfg.scale)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert swa.swa_device_error() == 0
    ref_o, ref_l = oracle.forward(q, k, v, cfg.win_left, cfg.win_right, cfg.dilation, 0, G.numpy(),
                                  cfg.scale)
    compare(out.float().cpu().numpy(), ref_o, BF16_MAX_ABS, BF16_MEAN_ABS, what="out")
    compare(lse.cpu().numpy(), ref_l, LSE_ABS, what="lse")


@pytest.mark.parametrize("case", [
    # (B, N, H, D, L, R, d, bs): D = 64, no GQA pair, short key walks
    (8, 4296, 16, 64, 100, 100, 1, 0),   # 34 query tiles per head, a ragged last one
    (8, 4296, 16, 64, 200, 0, 1, 0),     # causal
    (4, 8192, 16, 64, 64, 64, 2, 0),     # token dilation (two classes)
    (4, 8192, 16, 64, 128, 128, 2, 64),  # block dilation
])
def test_bf16_d64_mha_short_walks(swa, case):
    """D = 64 heads without a GQA pair (one head per CTA, two CTAs per SM)
    and walks of two to four key tiles, at batch sizes that fill many waves:
    sampled rows (tile, class and ragged-tail edges) against the oracle, and
    every output finite."""
    B, N, H, D, L, R, d, bs = case
    q, k, v = rand_case(B, N, H, H, D, 17)
    out, lse = run_forward(swa, q, k, v, L, R, d, bs, None, 0.0)
    edges = list(range(0, 4 * 128, 64)) + [N - 1, N - 129, N - 200, 4095, 4096, 4097]
    rows = sample_rows(B, H, N, 2500, seed=9, extra_i=edges)
    ref_o, ref_l = oracle.forward(q, k, v, L, R, d, bs, [], 0.0, rows=rows)
    compare(out[rows[:, 0], rows[:, 2], rows[:, 1]], ref_o, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare(lse[rows[:, 0], rows[:, 1], rows[:, 2]], ref_l, LSE_ABS, what="lse")
    assert np.isfinite(out).all() and np.isfinite(lse).all()
