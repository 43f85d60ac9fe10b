"""Parity of the grouped (mixture-of-experts) contraction with the oracle.

Layout: tokens routed to expert e occupy rows [start_e, start_e + count_e) of
the routed activations, each expert segment zero-padded to a multiple of 64
rows.  The three GEMMs of an expert FFN under the recipe:
  gate/up FPROP   Y_e  = X_e  W_gu,e^T      groups over token segments (ragged m)
  down DGRAD      dH_e = dY_e W_down,e      W_down stacked [E*2048, 1408] quantized
                                            ALONG_ROWS: expert e = K window e
  down WGRAD      dW_e = dY_e^T H_e         K = the expert's (padded) tokens
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_quantized_gemms_b200 import ufp4
from fp4_quantized_gemms_b200 import workloads as wl
from tests.gpu_util import GEMM_RTOL, needs_gpu, oracle_cfg, rel_fro, to_dev

pytestmark = needs_gpu

C, R = ufp4.ALONG_COLS, ufp4.ALONG_ROWS


def _routed(total, cols, std, seed, starts, counts):
    a = wl.normal(total, cols, std, seed)
    mask = np.zeros(total, dtype=bool)
    for s0, c in zip(starts, counts):
        mask[s0:s0 + c] = True
    a[~mask] = 0
    return a


def _moe(shape: wl.MoEShape, counts):
    starts, padded, total = wl.padded_offsets(counts, 64)
    E, Hd, F = shape.experts, shape.hidden, shape.ffn
    return dict(
        starts=starts, padded=padded, total=total, counts=counts,
        X=_routed(total, Hd, 1.0, 1, starts, counts),
        Wgu=wl.normal(E * 2 * F, Hd, 0.02, 2),
        dY=_routed(total, Hd, 1e-3, 3, starts, counts),
        Wd=wl.normal(E * Hd, F, 0.02, 4),
        H=_routed(total, F, 1.0, 5, starts, counts),
    )


def _quant(bits, axis, cfg):
    x = to_dev(bits)
    amax_d, amax_o = None, 0.0
    if cfg.scale_fmt == ufp4.SCALE_E4M3_X_FP32:
        amax_d = ufp4.rht_amax(x, axis, cfg.hadamard_n, cfg.rht_sign_mask)
        amax_o = oracle.rht_amax(bits, axis, cfg.hadamard_n, cfg.rht_sign_mask)
    return ufp4.rht_quantize(x, axis, cfg, tensor_amax=amax_d), amax_o


def _oracle_rows(bits, axis, cfg, amax, rows):
    oc = oracle_cfg(cfg)
    parts = [oracle.quantize(bits, axis, oc, tensor_amax=amax, r0=int(r), nr=1) for r in rows]
    return np.concatenate([p.dequantize() for p in parts])


def _run_gemm(name, d, cfgs, shape, sample_groups, per_group=6):
    """name in {fprop, dgrad, wgrad}: build operands and group table, run the
    grouped kernel, compare sampled entries of sampled groups with the oracle."""
    E, Hd, F = shape.experts, shape.hidden, shape.ffn
    starts, counts, padded = d["starts"], d["counts"], d["padded"]
    rt, sr0, sr1 = cfgs
    if name == "fprop":
        a_bits, a_ax, a_cfg = d["X"], C, rt
        b_bits, b_ax, b_cfg = d["Wgu"], C, rt
        groups = [(counts[e], 2 * F, Hd, starts[e], 0, e * 2 * F, 0, starts[e], 0) for e in range(E)]
        out_shape = (d["total"], 2 * F)
    elif name == "dgrad":
        a_bits, a_ax, a_cfg = d["dY"], C, sr0
        b_bits, b_ax, b_cfg = d["Wd"], R, rt
        groups = [(counts[e], F, Hd, starts[e], 0, 0, e * Hd, starts[e], 0) for e in range(E)]
        out_shape = (d["total"], F)
    else:
        a_bits, a_ax, a_cfg = d["dY"], R, sr1
        b_bits, b_ax, b_cfg = d["H"], R, rt
        groups = [(Hd, F, padded[e], 0, starts[e], 0, starts[e], e * Hd, 0) for e in range(E)]
        out_shape = (E * Hd, F)
    qa, amax_a = _quant(a_bits, a_ax, a_cfg)
    qb, amax_b = _quant(b_bits, b_ax, b_cfg)
    g = torch.tensor(np.array(groups, dtype=np.int64), device="cuda")
    out = torch.full(out_shape, float("nan"), dtype=torch.float32, device="cuda")
    ufp4.grouped_gemm(qa, qb, g, out)
    torch.cuda.synchronize()
    assert ufp4.check_device_status() == ufp4.OK
    got_all = out.cpu().numpy()
    rng = np.random.default_rng(5)
    n_h = a_cfg.hadamard_n
    inv_n = 1.0 / n_h if n_h else 1.0
    errs = []
    for e in sample_groups:
        m, n, k, ar, ac, br, bc, cr, cc = groups[e]
        if m == 0:
            continue
        ii = np.unique(np.concatenate([[0, m - 1], rng.choice(m, min(m, per_group), replace=False)]))
        jj = np.unique(np.concatenate([[0, n - 1], rng.choice(n, min(n, per_group), replace=False)]))
        A = _oracle_rows(a_bits, a_ax, a_cfg, amax_a, ar + ii)[:, ac:ac + k]
        B = _oracle_rows(b_bits, b_ax, b_cfg, amax_b, br + jj)[:, bc:bc + k]
        ref = oracle.gemm_dequantized(A, B, inv_n)
        got = got_all[np.ix_(cr + ii, cc + jj)]
        errs.append(rel_fro(got, ref))
        assert errs[-1] <= GEMM_RTOL, (name, e, errs[-1])
    # every output row that belongs to a group was written
    for (m, n, k, ar, ac, br, bc, cr, cc) in groups:
        assert not np.isnan(got_all[cr:cr + m, cc:cc + n]).any()
    return errs


def _cfgs(fmt, grid=0):
    rt = ufp4.QuantConfig(grid=grid, hadamard_n=16, block=16, scale_fmt=fmt)
    return rt, rt.with_(rounding=ufp4.ROUND_SR, sr_seed=1234, sr_stream=0), \
        rt.with_(rounding=ufp4.ROUND_SR, sr_seed=1234, sr_stream=1)


SMALL = wl.MoEShape(tokens=512, hidden=256, ffn=192, experts=8, topk=2, zipf_s=1.2)


@pytest.mark.parametrize("fmt,grid", [(ufp4.SCALE_FP32, ufp4.GRID_E1M2), (ufp4.SCALE_E4M3_X_FP32, ufp4.GRID_E1M2),
                                      (ufp4.SCALE_E4M3_X_FP32, ufp4.GRID_E2M1)])
@pytest.mark.parametrize("name", ["fprop", "dgrad", "wgrad"])
def test_grouped_small(fmt, grid, name):
    """8 experts, ragged counts (one expert empty), every group checked, for
    fp32 scales and for two-level scales on both grids."""
    counts = wl.moe_expert_counts(SMALL)
    counts[3] = 0                             # an expert with no tokens
    d = _moe(SMALL, counts)
    _run_gemm(name, d, _cfgs(fmt, grid), SMALL, range(SMALL.experts), per_group=40)


_FULL = {}


@pytest.mark.parametrize("fmt", [ufp4.SCALE_E4M3_X_FP32, ufp4.SCALE_FP32])
@pytest.mark.parametrize("name", ["fprop", "dgrad", "wgrad"])
def test_grouped_moe_config_sampled(fmt, name):
    """16384 tokens, top-6, 64 experts of FFN 1408 (gate/up 2816), hidden 2048,
    Zipf(1.2) counts: 98304 routed rows.  Largest, smallest and 4 random
    experts sampled."""
    if "d" not in _FULL:
        counts = wl.moe_expert_counts(wl.MOE)
        assert counts.sum() == wl.MOE.tokens * wl.MOE.topk
        _FULL["d"] = _moe(wl.MOE, counts)
    d = _FULL["d"]
    counts = d["counts"]
    rng = np.random.default_rng(1)
    sample = sorted(set([int(np.argmax(counts)), int(np.argmin(counts))] +
                        list(rng.choice(wl.MOE.experts, 4, replace=False))))
    _run_gemm(name, d, _cfgs(fmt), wl.MOE, sample)
