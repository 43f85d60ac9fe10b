"""Helpers for the GPU parity tests: move seeded inputs to the device, read the
library's packed outputs back in the oracle's logical layout."""
import numpy as np
import pytest
import torch

import oracle
from fp4_quantized_gemms_b200 import ufp4

needs_gpu = [pytest.mark.gpu,
             pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

GEMM_RTOL = 1e-5   # relative Frobenius error vs the fp64 oracle (the method's bound)


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit pattern (uint16) -> bf16 CUDA tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def oracle_cfg(cfg: ufp4.QuantConfig) -> oracle.QuantCfg:
    return oracle.QuantCfg(grid=cfg.grid, rounding=cfg.rounding, sr_seed=cfg.sr_seed,
                           sr_stream=cfg.sr_stream, hadamard_n=cfg.hadamard_n,
                           sign_mask=cfg.rht_sign_mask, block=cfg.block,
                           scale_fmt=cfg.scale_fmt)


def unpack_codes(q: ufp4.QTensor, rows=None) -> np.ndarray:
    """uint8 [rows, kpad/2] -> int8 nibbles [rows, kpad], low nibble first."""
    c = q.codes if rows is None else q.codes[torch.as_tensor(rows, device=q.codes.device)]
    b = c.cpu().numpy()
    out = np.empty((b.shape[0], b.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = b & 0x0F
    out[:, 1::2] = b >> 4
    return out


def logical_scales(q: ufp4.QTensor, rows=None) -> np.ndarray:
    """block-major [nblk, scale_ld] -> [rows, nblk]."""
    s = q.scales.cpu().numpy()[:, :q.rows].T
    return s if rows is None else s[np.asarray(rows)]


def tensor_scale(q: ufp4.QTensor) -> float:
    return float(q.tensor_scale.cpu().numpy()[0]) if q.tensor_scale is not None else 1.0


E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def expected_corr(codes: np.ndarray) -> np.ndarray:
    """E1M2 correction-plane nibbles from E1M2 code nibbles: magnitude k =
    e(k) + d(k) with e(k) the E2M1 value of the same bits, d(k) an E2M1 value
    (its code returned here), sign copied."""
    lut = np.zeros(16, dtype=np.int8)
    for nib in range(16):
        k, sign = nib & 7, nib & 8
        d = k - E2M1_VALUES[k]
        assert d in E2M1_VALUES, (k, d)
        lut[nib] = sign | E2M1_VALUES.index(d)
    return lut[codes.astype(np.int64) & 15]


def unpack_plane(t: torch.Tensor, rows=None) -> np.ndarray:
    c = t if rows is None else t[torch.as_tensor(rows, device=t.device)]
    b = c.cpu().numpy()
    out = np.empty((b.shape[0], b.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = b & 0x0F
    out[:, 1::2] = b >> 4
    return out


E4M3_OF_E1M2 = [0x00, 0x28, 0x30, 0x34, 0x38, 0x3A, 0x3C, 0x3E]   # E4M3 bytes of k/4, k = 0..7


def expected_elems8(codes: np.ndarray) -> np.ndarray:
    """MX element-plane bytes from E1M2 code nibbles: the OCP E4M3 encoding of
    +-k/4 (magnitude byte from the table, sign in bit 7)."""
    c = codes.astype(np.int64) & 15
    lut = np.array([E4M3_OF_E1M2[n & 7] | (0x80 if (n & 8) and (n & 7) else 0) for n in range(16)],
                   dtype=np.uint8)
    return lut[c]


def atoms_logical(q: ufp4.QTensor, rows=None) -> np.ndarray:
    """Factor atoms [ceil(rows/128), atoms_k, 512] -> [rows, slots]: byte
    16 (r % 32) + 4 ((r / 32) % 4) + s % 4 of atom (r / 128, s / 4) is the
    factor of K slot s of row r (slots of 16 elements for E4M3 factors, 32
    for UE8M0)."""
    w = 32 if q.cfg.scale_fmt == ufp4.SCALE_UE8M0 else 16
    slots = q.kpad // w
    r = np.arange(q.rows) if rows is None else np.asarray(rows)
    a = q.sf_atoms.cpu().numpy()
    s = np.arange(slots)
    byte = (16 * (r % 32) + 4 * ((r // 32) % 4))[:, None] + (s % 4)[None, :]
    return a[(r // 128)[:, None], (s // 4)[None, :], byte]


def lane_tiles_logical(q: ufp4.QTensor, rows=None) -> np.ndarray:
    """Per-lane factor tiles of an E1M2 operand with E4M3 factors
    ([ceil(rows/128)][ceil(kpad/128)][4096]) -> [rows, slots]: the
    factor of 16-slot s of row r is byte 2048 ((s / 4) % 2) + 16 L + 4 (L / 32)
    + s % 4 of tile (r / 128, s / 8), L = r % 128 (tensor-memory column
    4 ((s / 4) % 2) + L / 32 of lane L after one 128-lane copy)."""
    slots = q.kpad // 16
    r = np.arange(q.rows) if rows is None else np.asarray(rows)
    t = q.sf_lanes.cpu().numpy()
    s = np.arange(slots)
    L = (r % 128)[:, None]
    byte = 2048 * ((s // 4) % 2)[None, :] + 16 * L + 4 * (L // 32) + (s % 4)[None, :]
    return t[(r // 128)[:, None], (s // 8)[None, :], byte]


def assert_quant_equal(q: ufp4.QTensor, ref: oracle.QTensor, rows=None):
    if q.corr is not None:
        got_c = unpack_plane(q.corr, rows)
        want_c = expected_corr(ref.codes)
        if not np.array_equal(got_c, want_c):
            bad = np.argwhere(got_c != want_c)
            r, c = bad[0]
            raise AssertionError(f"{len(bad)} correction nibbles differ; first at ({r},{c}): gpu "
                                 f"{got_c[r, c]} expected {want_c[r, c]} (code {ref.codes[r, c]})")
    if q.elems8 is not None:
        e = q.elems8 if rows is None else q.elems8[torch.as_tensor(rows, device=q.elems8.device)]
        got_e = e.cpu().numpy()
        want_e = expected_elems8(ref.codes)
        if not np.array_equal(got_e, want_e):
            bad = np.argwhere(got_e != want_e)
            r, c = bad[0]
            raise AssertionError(f"{len(bad)} E4M3 element bytes differ; first at ({r},{c}): gpu "
                                 f"{got_e[r, c]:#x} expected {want_e[r, c]:#x} (code {ref.codes[r, c]})")
    got = unpack_codes(q, rows)
    if not np.array_equal(got, ref.codes):
        bad = np.argwhere(got != ref.codes)
        r, c = bad[0]
        raise AssertionError(f"{len(bad)} codes differ; first at ({r},{c}): gpu {got[r, c]} "
                             f"oracle {ref.codes[r, c]}")
    if q.sf_atoms is not None:
        w = 32 if q.cfg.scale_fmt == ufp4.SCALE_UE8M0 else 16
        want_a = ref.escales[:, (np.arange(q.kpad // w) * w) // q.cfg.block]
        got_a = atoms_logical(q, rows)
        if not np.array_equal(got_a, want_a):
            bad = np.argwhere(got_a != want_a)
            r, c = bad[0]
            raise AssertionError(f"{len(bad)} factor-atom bytes differ; first at (row {r}, slot {c}): gpu "
                                 f"{got_a[r, c]:#x} expected {want_a[r, c]:#x}")
    if q.sf_lanes is not None:
        want_l = ref.escales[:, (np.arange(q.kpad // 16) * 16) // q.cfg.block]
        got_l = lane_tiles_logical(q, rows)
        if not np.array_equal(got_l, want_l):
            bad = np.argwhere(got_l != want_l)
            r, c = bad[0]
            raise AssertionError(f"{len(bad)} per-lane tile factor bytes differ; first at (row {r}, slot {c}): "
                                 f"gpu {got_l[r, c]:#x} expected {want_l[r, c]:#x}")
    sc = logical_scales(q, rows)
    if ref.scales is not None:
        assert np.array_equal(sc.view(np.uint32), ref.scales.view(np.uint32)), "fp32 scales differ"
    else:
        assert np.array_equal(sc, ref.escales), "E4M3 block scales differ"
        assert np.float32(tensor_scale(q)) == np.float32(ref.S), "tensor scale differs"


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))
