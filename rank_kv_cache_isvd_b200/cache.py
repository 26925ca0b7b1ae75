"""Convenience wrapper over the C ABI: owns an ``iskv_handle`` and allocates caller-side buffers
with torch (device memory and streams only; all arithmetic runs in ``libiskv.so``)."""
from __future__ import annotations

import torch

from .binding import (ISKV_BF16, ISKV_F32, check, iskv_append_block, iskv_config, iskv_create,
                      iskv_decode_attn, iskv_destroy, iskv_fold_stats, iskv_get_factors,
                      iskv_append_decode, iskv_join, iskv_launch_count,
                      iskv_num_tokens, iskv_reconstruct, iskv_reset, iskv_storage_bytes,
                      iskv_sync_status)


class IsKVCache:
    """iS-KV cache of ``n_layers`` layers x ``batch`` sequences x ``n_kv_heads`` kv-heads."""

    def __init__(self, *, batch: int, n_layers: int, n_kv_heads: int, n_q_heads: int,
                 rank_k: int, rank_v: int, block: int, window: int, max_tokens: int,
                 kv_dtype: str = "bf16", rope: bool = True, rope_theta: float = 5e5,
                 rotate_history: bool = True, head_dim: int = 128,
                 lookahead_folds: bool = False, fixed_basis: bool = False,
                 coord_bf16: bool = False, prot_cap: int = 0, joint_heads: bool = False):
        self.cfg = iskv_config(batch, n_layers, n_kv_heads, n_q_heads, head_dim, rank_k, rank_v,
                               block, window, max_tokens,
                               ISKV_BF16 if kv_dtype == "bf16" else ISKV_F32, int(rope),
                               float(rope_theta), int(rotate_history), int(lookahead_folds),
                               int(fixed_basis), int(coord_bf16), int(prot_cap),
                               int(joint_heads))
        self.dtype = torch.bfloat16 if kv_dtype == "bf16" else torch.float32
        self.handle = 0
        code, h = iskv_create(self.cfg)
        check(code, "iskv_create")
        self.handle = h

    # -- lifetime ----------------------------------------------------------------------------
    def close(self) -> None:
        if self.handle:
            iskv_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- calls ---------------------------------------------------------------------------------
    def append(self, layer: int, k_rows: torch.Tensor, v_rows: torch.Tensor, stream=None) -> None:
        """``k_rows``/``v_rows``: ``[batch][n_kv][m][d]`` (or ``[L][batch][n_kv][m][d]`` with
        ``layer=-1``), contiguous, on the device, in the cache's kv dtype."""
        assert k_rows.dtype == self.dtype and v_rows.dtype == self.dtype
        assert k_rows.is_contiguous() and v_rows.is_contiguous()
        check(iskv_append_block(self.handle, layer, k_rows, v_rows, k_rows.shape[-2], stream),
              "iskv_append_block")

    def prefill(self, layer: int, k_rows: torch.Tensor, v_rows: torch.Tensor, protect=None,
                stream=None) -> None:
        """Prefill of an empty layer (``[batch][n_kv][T0][d]`` rows): exact window, protected
        rows, truncated SVD of the rest. ``protect``: ``(chunk, m, suffix, rho)`` or ``None``."""
        from .binding import iskv_prefill, iskv_protect
        assert k_rows.dtype == self.dtype and k_rows.is_contiguous() and v_rows.is_contiguous()
        pr = None if protect is None else iskv_protect(*protect)
        check(iskv_prefill(self.handle, layer, k_rows, v_rows, k_rows.shape[-2], pr, stream),
              "iskv_prefill")

    def decode(self, layer: int, q: torch.Tensor, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        assert q.dtype == torch.float32 and q.is_contiguous()
        if out is None:
            out = torch.empty_like(q)
        check(iskv_decode_attn(self.handle, layer, q, out, stream), "iskv_decode_attn")
        return out

    def append_decode(self, layer: int, k_row: torch.Tensor, v_row: torch.Tensor, q: torch.Tensor,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """One decode step: append one row per (sequence, kv-head) (``[batch][n_kv][1][d]``) and
        attend over every position including it."""
        assert k_row.dtype == self.dtype and k_row.is_contiguous() and v_row.is_contiguous()
        assert q.dtype == torch.float32 and q.is_contiguous()
        if out is None:
            out = torch.empty_like(q)
        check(iskv_append_decode(self.handle, layer, k_row, v_row, q, out, stream),
              "iskv_append_decode")
        return out

    def reconstruct(self, layer: int, which: int, apply_rope: bool = False,
                    stream=None) -> torch.Tensor:
        t = self.tokens(layer)
        out = torch.empty((self.cfg.batch, self.cfg.n_kv_heads, t, self.cfg.head_dim),
                          dtype=torch.float32, device="cuda")
        check(iskv_reconstruct(self.handle, layer, which, int(apply_rope), out, stream),
              "iskv_reconstruct")
        return out

    def factors(self, layer: int, seq: int, kv_head: int, which: int, stream=None):
        """``(coords [n_c][r], basis [d][r], sigma [r], k, n_c)`` copies of one unit."""
        r = self.cfg.rank_k if which == 0 else self.cfg.rank_v
        code, k, n_c = iskv_get_factors(self.handle, layer, seq, kv_head, which)
        check(code, "iskv_get_factors")
        coords = torch.empty((max(n_c, 1), r), dtype=torch.float32, device="cuda")
        basis = torch.empty((self.cfg.head_dim, r), dtype=torch.float32, device="cuda")
        sigma = torch.empty((r,), dtype=torch.float32, device="cuda")
        code, k, n_c = iskv_get_factors(self.handle, layer, seq, kv_head, which, coords, basis,
                                        sigma, stream)
        check(code, "iskv_get_factors")
        return coords[:n_c], basis, sigma, k, n_c

    def tokens(self, layer: int) -> int:
        code, t = iskv_num_tokens(self.handle, layer)
        check(code, "iskv_num_tokens")
        return t

    def storage_bytes(self, layer: int) -> int:
        code, b = iskv_storage_bytes(self.handle, layer)
        check(code, "iskv_storage_bytes")
        return b

    def join(self, stream=None) -> None:
        """Joins folds started ahead of time into ``stream`` (needed before ending a capture)."""
        check(iskv_join(self.handle, stream), "iskv_join")

    def reset(self, stream=None) -> None:
        check(iskv_reset(self.handle, stream), "iskv_reset")

    def launches(self) -> int:
        code, n = iskv_launch_count(self.handle)
        check(code, "iskv_launch_count")
        return n

    def fold_stats(self, stream=None):
        """``(max_sweeps, total_sweeps, cores)`` of the core SVDs since creation/reset."""
        code, m, t, c = iskv_fold_stats(self.handle, stream)
        check(code, "iskv_fold_stats")
        return m, t, c

    def status(self, stream=None) -> int:
        return iskv_sync_status(self.handle, stream)
