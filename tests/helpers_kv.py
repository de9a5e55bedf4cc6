"""Shared helpers of the GPU parity tests: cache construction through the CUDA library and
the oracle's view of the same seeded inputs.  Imported by tests only."""
from __future__ import annotations

import numpy as np

from oracle import attention as oatt
from oracle import layout as olay
from oracle import quant as oq

ATOL = 2e-3      # max abs error on fp32 outputs (the target's tolerance)
RTOL_GATE = 2e-3  # internal gate on ||o_gpu - o_ref|| / ||o_ref||


def torch_mod():
    import torch

    return torch


def lib():
    from quantized_paged_kv_q4_b200 import kvattn

    return kvattn


class GpuCache:
    """Device page pools for one layer (H_kv units) filled through kvattn_quantize_append."""

    def __init__(self, H_kv, H_q, n_blocks, v_fmt="q4_0", n_phys=None, perm=None, device="cuda", k_fmt="q8_0"):
        torch = torch_mod()
        kv = lib()
        self.H_kv, self.H_q, self.n_blocks, self.v_fmt, self.k_fmt = H_kv, H_q, n_blocks, v_fmt, k_fmt
        self.n_phys = n_phys or H_kv * n_blocks
        kb = olay.page_bytes("k", k_fmt)
        vb = olay.page_bytes("v", v_fmt)
        self.k_pool = torch.zeros((self.n_phys, kb), dtype=torch.uint8, device=device)
        self.v_pool = torch.zeros((self.n_phys, vb), dtype=torch.uint8, device=device)
        if perm is None:
            perm = np.arange(self.n_phys, dtype=np.int32)
        self.page_table_np = np.asarray(perm[: H_kv * n_blocks], dtype=np.int32).reshape(H_kv, n_blocks)
        self.page_table = torch.from_numpy(self.page_table_np.copy()).to(device)
        self.desc = kv.make_desc(H_kv, H_q, self.k_pool, self.v_pool, self.n_phys, v_fmt=v_fmt, k_fmt=k_fmt)

    def append(self, k, v, pos0):
        """k, v: fp32 arrays [n][H_kv][256] (numpy or torch)."""
        torch = torch_mod()
        kt = torch.as_tensor(np.ascontiguousarray(k) if isinstance(k, np.ndarray) else k).to("cuda").contiguous()
        vt = torch.as_tensor(np.ascontiguousarray(v) if isinstance(v, np.ndarray) else v).to("cuda").contiguous()
        lib().kvattn_quantize_append(self.desc, kt, vt, kt.shape[0], pos0, self.page_table, self.n_blocks)


class OracleCache:
    """The oracle's quantised view of one layer: codes and scales per unit and token."""

    def __init__(self, k, v, v_fmt="q4_0", k_fmt="q8_0"):
        # k, v: fp32 [T][H_kv][256]
        self.v_fmt, self.k_fmt = v_fmt, k_fmt
        self.kc, self.kd = oq.quantize(np.asarray(k, np.float32), k_fmt)        # [T][H][8][32], [T][H][8]
        self.vc, self.vd = oq.quantize(np.asarray(v, np.float32), v_fmt)
        self.T = k.shape[0]

    def khat(self, h):
        return oq.dequantize(self.kc[:, h], self.kd[:, h], self.k_fmt)

    def vhat(self, h):
        return oq.dequantize(self.vc[:, h], self.vd[:, h], self.v_fmt)

    @staticmethod
    def _unwritten(fmt):
        """Codes of slots never written (zero bytes in a zero-filled pool: Q8_0 stores q + 128)."""
        if fmt == "q8_0":
            return np.full((128, 8, 32), -128, np.int8)
        return np.zeros((128, 8, 32), np.uint8)

    def page_bytes(self, h, blk, role):
        """Expected bytes of logical block `blk` of unit h (slots beyond T stay zero bytes)."""
        a, b = blk * 128, min((blk + 1) * 128, self.T)
        if role == "k":
            codes = self._unwritten(self.k_fmt)
            d = np.zeros((128,) + self.kd.shape[2:], np.float16)  # (d, m) pairs for Q5_1
            codes[: b - a] = self.kc[a:b, h]
            d[: b - a] = self.kd[a:b, h]
            return olay.encode_page("k", self.k_fmt, codes, d)
        codes = self._unwritten(self.v_fmt)
        d = np.zeros((128,) + self.vd.shape[2:], np.float16)  # (d, m) pairs for Q4_1
        codes[: b - a] = self.vc[a:b, h]
        d[: b - a] = self.vd[a:b, h]
        return olay.encode_page("v", self.v_fmt, codes, d)

    def attend(self, q, q_pos, h, group, key_idx=None):
        """q: [n_q][H_q][256]; returns (o [n_q][group][256], lse [n_q][group]) for KV head h."""
        n_q = q.shape[0]
        rows = np.concatenate([q[i, h * group:(h + 1) * group] for i in range(n_q)], 0)
        qp = np.repeat(np.asarray(q_pos), group)
        kh, vh = self.khat(h), self.vhat(h)
        pos = np.arange(self.T)
        if key_idx is not None:
            kh, vh, pos = kh[key_idx], vh[key_idx], pos[key_idx]
        o, l = oatt.attend(rows, kh, vh, pos, qp, 1.0 / 16.0)
        return o.reshape(n_q, group, -1), l.reshape(n_q, group)


def compare(o_gpu, lse_gpu, o_ref, lse_ref):
    """Asserts the tolerance (ATOL absolute on every output and on lse, plus the relative
    gate); returns (max_abs, rel, lse_abs)."""
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    err = np.abs(o_gpu - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    lg, lr = np.asarray(lse_gpu, np.float64), np.asarray(lse_ref, np.float64)
    assert np.array_equal(np.isneginf(lg), np.isneginf(lr)), "masked rows differ"
    fin = np.isfinite(lr)
    lse_abs = float(np.abs(lg[fin] - lr[fin]).max()) if fin.any() else 0.0
    assert max_abs <= ATOL, f"max abs error {max_abs} (tolerance {ATOL})"
    assert rel <= RTOL_GATE, f"relative error {rel}"
    assert lse_abs <= ATOL, f"lse error {lse_abs}"
    return max_abs, rel, lse_abs
