"""Test support: run one step of a workload through the library on the GPU and
through the CPU oracle on the same seeded inputs.

Context rows of the requests the oracle checks come from the host generator
(workloads.Workload.ctx_rows); the other requests' context is drawn on the
GPU (seeded torch generator) so that full-size launches stay cheap to set up.
Their values never reach a compared output: attention of request r reads
only request r's pages.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from workloads import BF16_NAN, Workload

NAN_BITS = int(BF16_NAN)


def dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def nan_pool(w: Workload) -> torch.Tensor:
    return torch.full(w.pool_shape(), float("nan"), dtype=torch.bfloat16, device="cuda")


class DeviceStep:
    """Device buffers of one workload: pools filled with context, the step's
    new rows, queries and metadata."""

    def __init__(self, pkv, w: Workload, host_ids=None, fill_seed: int = 1234):
        self.pkv, self.w = pkv, w
        host_ids = list(range(w.B)) if host_ids is None else sorted(set(int(r) for r in host_ids))
        self.host_ids = host_ids
        self.k_pool, self.v_pool = nan_pool(w), nan_pool(w)
        self.page_table = dev_i32(w.page_table)
        self.kv_lens = dev_i32(w.kv_lens)
        others = [r for r in range(w.B) if r not in set(host_ids)]
        if others:
            self._device_fill(others, fill_seed)
        if host_ids:
            k, v, s = w.batch_ctx(host_ids)
            if len(s):
                pkv.pkv_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(s), self.k_pool, self.v_pool)
        # this step's new rows and queries (small: host-generated for all)
        k, v, s = w.batch_new()
        self.k_new, self.v_new, self.slots_new = dev_bf16(k), dev_bf16(v), dev_i32(s)
        dec, pre = w.decode_ids, w.prefill_ids
        self.q_dec = dev_bf16(w.batch_q(dec)) if len(dec) else None
        self.q_pre = dev_bf16(w.batch_q(pre)) if len(pre) else None
        self.cu_q = dev_i32(w.cu_q_lens(pre)) if len(pre) else None
        self.ctx_pre = dev_i32(w.ctx_lens[pre]) if len(pre) else None
        self.pt_dec = dev_i32(w.page_table[dec]) if len(dec) else None
        self.pt_pre = dev_i32(w.page_table[pre]) if len(pre) else None
        self.len_dec = dev_i32(w.kv_lens[dec]) if len(dec) else None
        torch.cuda.synchronize()

    def _device_fill(self, ids, seed):
        w = self.w
        gen = torch.Generator(device="cuda").manual_seed(seed)
        # in groups of requests, to bound the fp32 temporaries
        group, budget = [], 0
        for r in ids + [None]:
            if r is not None:
                group.append(r)
                budget += int(w.ctx_lens[r])
            if group and (r is None or budget > (1 << 18)):
                slots = w.ctx_slots(group)
                n = len(slots)
                if n:
                    k = torch.randn((n, w.num_kv_heads, w.head_dim), generator=gen, device="cuda")
                    if w.k_rms_norm:
                        k = k / k.pow(2).mean(-1, keepdim=True).sqrt()
                    v = torch.randn((n, w.num_kv_heads, w.head_dim), generator=gen, device="cuda")
                    self.pkv.pkv_kv_append(k.bfloat16().contiguous(), v.bfloat16().contiguous(),
                                           dev_i32(slots), self.k_pool, self.v_pool)
                group, budget = [], 0

    # ---------------------------------------------------------------- steps
    def append(self):
        self.pkv.pkv_kv_append(self.k_new, self.v_new, self.slots_new, self.k_pool, self.v_pool)

    def decode(self, partition=0, workspace=None, out=None, out_lse=None):
        w = self.w
        return self.pkv.pkv_paged_attn_decode(
            self.q_dec, self.k_pool, self.v_pool, self.pt_dec, self.len_dec, w.scale,
            partition_tokens=partition, workspace=workspace, out=out, out_lse=out_lse)

    def prefill(self, out=None):
        w = self.w
        pre = w.prefill_ids
        return self.pkv.pkv_paged_attn_chunked_prefill(
            self.q_pre, self.cu_q, self.ctx_pre, self.k_pool, self.v_pool, self.pt_pre, w.scale,
            int(w.new_lens[pre].max()), out=out)


class OracleStep:
    """The oracle's view of the same step, restricted to ``ids``: a compact
    pool holding only those requests' pages (the oracle's output does not
    depend on where pages sit in the pool)."""

    def __init__(self, w: Workload, ids=None):
        ids = list(range(w.B)) if ids is None else sorted(set(int(r) for r in ids))
        self.w, self.ids = w, ids
        used = np.unique(np.concatenate([w.page_table[r][w.page_table[r] >= 0] for r in ids]))
        remap = np.full(w.num_pages, -1, np.int64)
        remap[used] = np.arange(len(used))
        table = np.full_like(w.page_table, -1)
        for r in ids:
            row = w.page_table[r]
            table[r, row >= 0] = remap[row[row >= 0]]
        self.used_pages = used
        self.cw = Workload(w.name, w.seed, w.num_q_heads, w.num_kv_heads, w.head_dim,
                           w.page_size, len(used), table, w.ctx_lens, w.new_lens, w.is_prefill,
                           w.k_rms_norm)
        self.k_pool = self.cw.empty_pool()
        self.v_pool = self.cw.empty_pool()
        k, v, s = self.cw.batch_ctx(ids)
        oracle.kv_append(self.k_pool, self.v_pool, k, v, s, w.page_size)

    def append(self):
        k, v, s = self.cw.batch_new(self.ids)
        oracle.kv_append(self.k_pool, self.v_pool, k, v, s, self.w.page_size)

    def decode(self):
        """(out, lse) for the decode requests among ids, indexed like decode_ids."""
        w = self.w
        dec = list(w.decode_ids)
        q = np.zeros((len(dec), w.num_q_heads, w.head_dim), np.uint16)
        sel = [i for i, r in enumerate(dec) if r in set(self.ids)]
        for i in sel:
            q[i] = w.q_rows(dec[i])[0]
        out, lse = oracle.decode_attention(q, self.k_pool, self.v_pool, self.cw.page_table[dec],
                                           w.kv_lens[dec], w.page_size, w.scale, ids=sel)
        return out, lse, sel

    def prefill(self):
        w = self.w
        pre = list(w.prefill_ids)
        cu = w.cu_q_lens(pre)
        q = np.zeros((int(cu[-1]), w.num_q_heads, w.head_dim), np.uint16)
        sel = [i for i, r in enumerate(pre) if r in set(self.ids)]
        for i in sel:
            q[cu[i]:cu[i + 1]] = w.q_rows(pre[i])
        out, lse = oracle.chunked_prefill_attention(q, cu, w.ctx_lens[pre], self.k_pool, self.v_pool,
                                                    self.cw.page_table[pre], w.page_size, w.scale,
                                                    ids=sel)
        rows = np.concatenate([np.arange(cu[i], cu[i + 1]) for i in sel]) if sel else np.zeros(0, int)
        return out, lse, rows


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


MAX_ABS, MEAN_ABS = 1e-2, 1e-3


def assert_close(got: np.ndarray, ref: np.ndarray, what: str):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3g} > {MAX_ABS}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3g} > {MEAN_ABS}"
    return float(err.max()), float(err.mean())
