"""Lay a synthetic workload out in the block pool and on the device, and run
one decode step through the C ABI.

A workload (see the ``synth`` package) supplies the random draws: the free
list order, the pool operations to replay (create / append / fork / release),
and the logical K/V/q values of every sequence.  This module replays the
operations on the C++ pool, writes every token that precedes the step into
the device cache with ``pa_write_kv`` (and runs the copy-on-write copies the
pool queued with ``pa_copy_blocks``), then prepares the step: one new token
per sequence (slot mapping from the pool), the block table, the lengths and
the queries.  Slots and blocks no token has written hold a bf16 NaN poison so
that any read of unused storage shows up in the outputs.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from ._abi import (pa_copy_blocks, pa_copy_blocks_fp8, pa_decode, pa_decode_fp8, pa_decode_fp8_workspace_bytes,
                   pa_decode_workspace_bytes, pa_write_kv, pa_write_kv_fp8)
from .pool import BlockPool

POISON_BITS = 0x7FC1  # a bf16 quiet NaN
POISON_FP8 = 0x7F  # the e4m3 NaN code


def to_device_bf16(a: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns -> a bf16 CUDA tensor (bit copy)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 bit patterns on the host."""
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@dataclasses.dataclass
class DeviceStep:
    pool: BlockPool
    ids: list
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    caches: list  # [(k_cache, v_cache)] per layer, bf16 [NB, B, H_kv, D]
    q: torch.Tensor  # [S, H_q, D] bf16
    k_new: torch.Tensor  # [S, H_kv, D] bf16: the step's token
    v_new: torch.Tensor
    slot_mapping: torch.Tensor  # [S] int64
    cow_pairs: torch.Tensor  # [P, 2] int64 (copies queued by the step's appends)
    block_tables: torch.Tensor  # [S, W] int32
    seq_lens: torch.Tensor  # [S] int32 (after the step's token)
    max_seq_len: int
    scale: float
    out: torch.Tensor  # [S, H_q, D] bf16
    workspace: torch.Tensor | None
    # host copies, for checks
    block_tables_np: np.ndarray
    seq_lens_np: np.ndarray
    slot_mapping_np: np.ndarray
    cow_pairs_np: np.ndarray
    history_pairs_np: np.ndarray
    kv_dtype: str = "bf16"
    k_scale: float = 1.0
    v_scale: float = 1.0


def _write_rows(w, pool, kc, vc, items, device, chunk_tokens=1 << 16, fp8_scales=None):
    """Write logical rows (sid, a, b) at the pool's slots, in chunks."""
    buf_k, buf_v, buf_s, n = [], [], [], 0

    def flush():
        nonlocal buf_k, buf_v, buf_s, n
        if n:
            k = to_device_bf16(np.concatenate(buf_k), device)
            v = to_device_bf16(np.concatenate(buf_v), device)
            s = torch.from_numpy(np.concatenate(buf_s)).to(device)
            if fp8_scales is None:
                pa_write_kv(k, v, s, kc, vc)
            else:
                pa_write_kv_fp8(k, v, s, kc, vc, *fp8_scales)
        buf_k, buf_v, buf_s, n = [], [], [], 0

    for sid, a, b in items:
        if b <= a:
            continue
        buf_k.append(w.rows("k", sid, a, b))
        buf_v.append(w.rows("v", sid, a, b))
        buf_s.append(pool.slots(sid, a, b - a))
        n += b - a
        if n >= chunk_tokens:
            flush()
    flush()


def stage(w, device="cuda", layers: int = 1, rule: str = "shared", poison: bool = True,
          kv_dtype: str = "bf16", k_scale: float = 1.0 / 64, v_scale: float = 1.0 / 64) -> DeviceStep:
    """kv_dtype "bf16" (default) or "fp8" (E4M3 codes, value = code * scale)."""
    sh = w.shape
    pool = BlockPool(sh.num_blocks, sh.block_size, w.free_order, rule)
    w.ops(pool)
    shape = (sh.num_blocks, sh.block_size, sh.num_kv_heads, sh.head_dim)
    fp8 = kv_dtype == "fp8"
    if fp8:
        fill = POISON_FP8 if poison else 0
        kc = torch.full(shape, fill, dtype=torch.uint8, device=device)
        vc = torch.full(shape, fill, dtype=torch.uint8, device=device)
        scales = (k_scale, v_scale)
    else:
        fill = POISON_BITS if poison else 0
        kc = torch.full(shape, fill, dtype=torch.int16, device=device).view(torch.bfloat16)
        vc = torch.full(shape, fill, dtype=torch.int16, device=device).view(torch.bfloat16)
        scales = None

    if w.shared_len:
        _write_rows(w, pool, kc, vc, [(w.seq_ids[0], 0, w.shared_len)], device, fp8_scales=scales)
    if w.suffix_ops is not None:
        w.suffix_ops(pool)
    hist_pairs = pool.take_cow_pairs()
    if len(hist_pairs):
        (pa_copy_blocks_fp8 if fp8 else pa_copy_blocks)(kc, vc, torch.from_numpy(hist_pairs).to(device))
    _write_rows(w, pool, kc, vc,
                [(sid, w.shared_len, pool.seq_len(sid)) for sid in w.seq_ids], device, fp8_scales=scales)

    # the step: one new token per sequence
    for sid in w.seq_ids:
        if not pool.append(sid, w.step_tokens):
            raise RuntimeError("pool has no room for the step's tokens")
    pairs = pool.take_cow_pairs()
    slots = pool.step_slots(w.seq_ids, w.step_tokens)
    lens = pool.seq_lens(w.seq_ids)
    width = max(1, max(pool.num_blocks_of(s) for s in w.seq_ids))
    bt = pool.block_table(w.seq_ids, width)
    k_new = np.stack([w.rows("k", sid, int(n) - 1, int(n))[0] for sid, n in zip(w.seq_ids, lens)])
    v_new = np.stack([w.rows("v", sid, int(n) - 1, int(n))[0] for sid, n in zip(w.seq_ids, lens)])

    caches = [(kc, vc)] + [(kc.clone(), vc.clone()) for _ in range(layers - 1)]
    S = len(w.seq_ids)
    q = to_device_bf16(w.q, device)
    max_len = int(lens.max()) if S else 0
    if fp8:
        need = pa_decode_fp8_workspace_bytes(S, sh.num_q_heads, max_len, kc, vc, k_scale, v_scale)
    else:
        need = pa_decode_workspace_bytes(S, sh.num_q_heads, max_len, kc, vc)
    ws = torch.empty(need, dtype=torch.uint8, device=device) if need else None
    return DeviceStep(
        pool=pool, ids=list(w.seq_ids), num_q_heads=sh.num_q_heads, num_kv_heads=sh.num_kv_heads,
        head_dim=sh.head_dim, block_size=sh.block_size, num_blocks=sh.num_blocks, caches=caches,
        q=q, k_new=to_device_bf16(k_new, device), v_new=to_device_bf16(v_new, device),
        slot_mapping=torch.from_numpy(slots).to(device),
        cow_pairs=torch.from_numpy(np.ascontiguousarray(pairs.reshape(-1, 2))).to(device),
        block_tables=torch.from_numpy(bt).to(device), seq_lens=torch.from_numpy(lens).to(device),
        max_seq_len=max_len, scale=w.scale, out=torch.empty_like(q), workspace=ws,
        block_tables_np=bt, seq_lens_np=lens, slot_mapping_np=slots,
        cow_pairs_np=pairs.reshape(-1, 2), history_pairs_np=hist_pairs.reshape(-1, 2),
        kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale)


def run_step(st: DeviceStep, layer: int = 0, stream=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """One decode step on one layer: queued copies, the step's KV write, decode."""
    kc, vc = st.caches[layer]
    out = st.out if out is None else out
    if st.kv_dtype == "fp8":
        if st.cow_pairs.shape[0]:
            pa_copy_blocks_fp8(kc, vc, st.cow_pairs, stream=stream)
        pa_write_kv_fp8(st.k_new, st.v_new, st.slot_mapping, kc, vc, st.k_scale, st.v_scale, stream=stream)
        return pa_decode_fp8(st.q, kc, vc, st.k_scale, st.v_scale, st.block_tables, st.seq_lens, st.scale,
                             out=out, max_seq_len=st.max_seq_len, workspace=st.workspace, stream=stream)
    if st.cow_pairs.shape[0]:
        pa_copy_blocks(kc, vc, st.cow_pairs, stream=stream)
    pa_write_kv(st.k_new, st.v_new, st.slot_mapping, kc, vc, stream=stream)
    return pa_decode(st.q, kc, vc, st.block_tables, st.seq_lens, st.scale, out=out,
                     max_seq_len=st.max_seq_len, workspace=st.workspace, stream=stream)
