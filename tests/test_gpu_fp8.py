"""GPU parity of the fp8 (e4m3) Q K^T path: the quantised tiles and their scales bit for bit,
and the attention against the oracle's fp8 model (Q, K quantised per tile, exact fp64 after)."""
import numpy as np
import pytest

import oracle.vsa_oracle as O
from gpu_util import LayerRun, bf16_to_f64, check_close, oracle_inputs_f64, ragged_gpu_config
from vsa_synth import get_config

pytestmark = pytest.mark.gpu

CASES = {
    "ragged128": (lambda: ragged_gpu_config(128), 0.5),
    "ragged128_tripool": (lambda: ragged_gpu_config(128, "tripool", seed=25), 0.5),
    "medium": (lambda: get_config("medium").with_(heads=6, tile_shapes=get_config("medium").tile_shapes[:6]), 0.75),
}

_runs = {}


def run(name):
    import torch
    if name not in _runs:
        make, s = CASES[name]
        r = LayerRun(make(), s).run(fused=True)
        f8 = r.plan.allocate_fp8()
        b = r.bufs
        r.plan.tile_pack_pool_fp8(r.q, r.k_t, r.v, b["qp"], b["kp"], b["vp"], f8["qp8"], f8["kp8"],
                                  f8["q_scale"], f8["k_scale"], b["workspace"])
        op8 = torch.zeros_like(b["op"])
        r.plan.sparse_attn_fp8(f8["qp8"], f8["kp8"], f8["q_scale"], f8["k_scale"], b["vp"], b["idx"], op8)
        out8 = torch.empty_like(r.out)
        r.plan.tile_unpack(op8, out8)
        r.plan.check()
        _runs[name] = (r, f8, out8)
    return _runs[name]


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_tiles_and_scales_bit_exact(name):
    import torch
    r, f8, _ = run(name)
    cfg = r.cfg
    q, k, v = oracle_inputs_f64(r.inp)
    nt = r.plan.info.nt_max
    shape = (cfg.batch, cfg.heads, nt, 64, cfg.head_dim)
    got = {"q": f8["qp8"].view(shape).cpu().numpy(), "k": f8["kp8"].view(shape).cpu().numpy()}
    sc = {"q": f8["q_scale"].view(cfg.batch, cfg.heads, nt).cpu().numpy(),
          "k": f8["k_scale"].view(cfg.batch, cfg.heads, nt).cpu().numpy()}
    for name_t, x in (("q", q), ("k", k)):
        for b in range(cfg.batch):
            for h in range(cfg.heads):
                til = O.head_tiling(cfg, h)
                for n, toks in enumerate(til.all):
                    codes, scale = O.quantize_tile_e4m3(x[b, toks, h])
                    assert np.float32(sc[name_t][b, h, n]) == np.float32(scale), (name_t, b, h, n)
                    want = torch.from_numpy(codes).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                    assert np.array_equal(got[name_t][b, h, n, :len(toks)], want), (name_t, b, h, n)
                    assert not np.any(got[name_t][b, h, n, len(toks):]), (name_t, b, h, n)


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_attention_matches_oracle_model(name):
    r, _, out8 = run(name)
    q, k, v = oracle_inputs_f64(r.inp)
    kept = {(b, h): r.kept(b, h) for b in range(r.cfg.batch) for h in range(r.cfg.heads)}
    res = O.run_layer(r.cfg, q, k, v, r.k, gate=r.inp.gate, w_q=r.inp.w_q, w_k=r.inp.w_k, kept=kept, qk_fp8=True)
    check_close(bf16_to_f64(out8), res.out)


def test_fp8_needs_head_dim_128():
    import tile_sparse_video_pack_b200 as T
    r = LayerRun(get_config("tiny"), 0.5).run(fused=True)
    f8 = r.plan.allocate_fp8()
    with pytest.raises(T.vsa.VsaError, match="UNSUPPORTED"):
        r.plan.sparse_attn_fp8(f8["qp8"], f8["kp8"], f8["q_scale"], f8["k_scale"], r.bufs["vp"], r.bufs["idx"],
                               r.bufs["op"])
