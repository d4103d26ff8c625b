"""D paged KV shards on one GPU, driven through the C ABI.

``ShardedPagedCache`` owns the device buffers of one decode problem: the D
shard pools, their block tables, the per-shard partial outputs, the merged
output and the workspace.  torch only allocates memory here; the tables are
built by ``dcp_build_block_table`` (interleaved or contiguous-chunk rule), the
cache write is ``dcp_place_kv`` (bf16 pools, or FP8 E4M3 codes with per-tensor
scales), and a decode step is ``dcp_decode_partial_all`` (or D
``dcp_decode_partial`` calls) followed by ``dcp_lse_merge``.  With ``q_len > 1``
each request decodes ``q_len`` draft tokens (causal within the draft) and the
outputs gain a ``q_len`` axis.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from . import dcp


class ShardedPagedCache:
    def __init__(self, layout: int, num_q_heads: int, num_kv_heads: int, head_dim_qk: int, head_dim_v: int,
                 block_size: int, D: int, seq_lens: Sequence[int], softmax_scale: float, perm_seed: int = 0,
                 device="cuda", pool_fill: Optional[int] = None, q_len: int = 1, kv_dtype: int = 0,
                 k_scale: float = 1.0, v_scale: float = 1.0, shard_rule: int = 0):
        self.D = D
        self.q_len = q_len
        self.device = torch.device(device)
        self.seq_lens = [int(x) for x in seq_lens]
        self.batch = len(self.seq_lens)
        mlb, num_pages = dcp.dcp_block_table_extent(self.seq_lens, block_size, D, shard_rule)
        self.max_local_blocks = max(1, mlb)
        self.num_pages = num_pages
        self.tables_host, self.local_len = dcp.dcp_build_block_table(self.seq_lens, block_size, D, perm_seed,
                                                                     self.max_local_blocks, shard_rule)
        self.desc = dcp.make_desc(layout, self.batch, num_q_heads, num_kv_heads, head_dim_qk, head_dim_v,
                                  block_size, self.max_local_blocks, softmax_scale, q_len, kv_dtype, k_scale,
                                  v_scale, shard_rule)
        self.page_bytes = dcp.dcp_kv_page_bytes(self.desc)
        if self.page_bytes == 0:
            raise ValueError("unsupported attention shape")
        self.pools = []
        for s in range(D):
            n = max(1, int(num_pages[s])) * self.page_bytes // 2
            if pool_fill is None:
                self.pools.append(torch.empty(n, dtype=torch.int16, device=self.device))
            else:
                self.pools.append(torch.full((n,), pool_fill - (1 << 16) if pool_fill >= (1 << 15) else pool_fill,
                                             dtype=torch.int16, device=self.device))
        self.pool_pages = np.ascontiguousarray(num_pages, dtype=np.int32)
        self.tables = [torch.from_numpy(self.tables_host[s]).to(self.device) for s in range(D)]
        self.seq_lens_dev = torch.tensor(self.seq_lens, dtype=torch.int32, device=self.device)
        cu = np.zeros(self.batch + 1, dtype=np.int64)
        cu[1:] = np.cumsum(self.seq_lens)
        self.cu_seqlens = torch.from_numpy(cu).to(self.device)
        self.ws_bytes = dcp.dcp_decode_workspace_bytes(self.desc, D)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        dcp.dcp_workspace_init(self.workspace)
        # outputs [B][Hq](...) for single-token decode, [B][q_len][Hq](...) for multi-token decode
        rows = (self.batch, num_q_heads) if q_len == 1 else (self.batch, q_len, num_q_heads)
        self.O_parts = torch.empty((D, *rows, head_dim_v), dtype=torch.float32, device=self.device)
        self.LSE_parts = torch.empty((D, *rows), dtype=torch.float32, device=self.device)
        self.O = torch.empty((*rows, head_dim_v), dtype=torch.float32, device=self.device)
        self.LSE = torch.empty(rows, dtype=torch.float32, device=self.device)

    # ------------------------------------------------------------------ cache write
    def place(self, kv_src: torch.Tensor, device_error: Optional[torch.Tensor] = None) -> None:
        dcp.dcp_place_kv(self.desc, self.D, kv_src, self.cu_seqlens, self.seq_lens_dev, self.tables, self.pools,
                         self.pool_pages, device_error)

    # ------------------------------------------------------------------ decode
    def partials(self, q: torch.Tensor, per_shard: bool = False) -> None:
        if per_shard:
            for s in range(self.D):
                dcp.dcp_decode_partial(self.desc, q, self.pools[s], int(self.pool_pages[s]), self.tables[s],
                                       self.seq_lens_dev, s, self.D, self.O_parts[s], self.LSE_parts[s],
                                       self.workspace)
        else:
            dcp.dcp_decode_partial_all(self.desc, q, self.pools, self.pool_pages, self.tables, self.seq_lens_dev,
                                       self.D, list(self.O_parts), list(self.LSE_parts), self.workspace)

    def merge(self, with_lse: bool = True) -> None:
        rows = self.batch * self.q_len * self.desc.num_q_heads
        dcp.dcp_lse_merge(list(self.O_parts), list(self.LSE_parts), self.D, rows, self.desc.head_dim_v, self.O,
                          self.LSE if with_lse else None)

    def step(self, q: torch.Tensor, per_shard: bool = False):
        """One decode step: all shard partials, then the merge. Returns (O, LSE) device tensors."""
        self.partials(q, per_shard)
        self.merge()
        return self.O, self.LSE

    def device_error(self) -> int:
        return dcp.dcp_read_device_error(self.workspace)

    @property
    def kv_bytes(self) -> int:
        """KV bytes the method reads per step (tokens x bytes per token; padding excluded)."""
        d = self.desc
        eb = 1 if d.kv_dtype == dcp.DCP_KV_FP8_E4M3 else 2
        per = 2 * d.num_kv_heads * d.head_dim_qk * eb if d.layout == dcp.DCP_LAYOUT_GQA else d.head_dim_qk * eb
        return int(sum(self.seq_lens)) * per


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class HostStepPipeline:
    """Decode steps fed from, and returned to, pinned host memory.

    Per step there is one host-to-device copy of the step's packed inputs (the
    query, the sequence lengths and the D block tables) and one device-to-host
    copy of its packed results (O and LSE).  Two buffer sets alternate between
    steps and three streams (upload, compute, download) are ordered with
    events, so step i's inputs upload while step i-1 computes and step i-1's
    results download while step i computes.  The compute itself is
    ``dcp_decode_partial_all`` + ``dcp_lse_merge`` on the cache's pools.
    """

    def __init__(self, cache: ShardedPagedCache):
        self.cache = c = cache
        d = c.desc
        self.rows = c.batch * c.q_len * d.num_q_heads  # (request, query token, head) rows
        self.q_elems = self.rows * d.head_dim_qk
        self.q_off, self.sl_off = 0, _align(self.q_elems * 2)
        self.tab_off = self.sl_off + _align(c.batch * 4)
        self.tab_elems = c.batch * c.max_local_blocks
        self.in_bytes = self.tab_off + c.D * self.tab_elems * 4
        self.o_elems = self.rows * d.head_dim_v
        self.lse_off = self.o_elems * 4
        self.out_bytes = self.lse_off + self.rows * 4
        dev = c.device
        self.dev_in = [torch.empty(self.in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.dev_out = [torch.empty(self.out_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_comp = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]

    # ------------------------------------------------------------------ host buffers
    def pack_inputs(self, q_bits, seq_lens, tables_host) -> torch.Tensor:
        """Pinned host buffer holding one step's inputs in the device layout."""
        buf = torch.zeros(self.in_bytes, dtype=torch.uint8).pin_memory()
        a = buf.numpy()
        a[self.q_off:self.q_off + self.q_elems * 2] = np.ascontiguousarray(q_bits).view(np.uint8).ravel()
        a[self.sl_off:self.sl_off + self.cache.batch * 4] = np.ascontiguousarray(seq_lens, np.int32).view(np.uint8)
        a[self.tab_off:] = np.ascontiguousarray(tables_host, np.int32).view(np.uint8).ravel()
        return buf

    def host_output(self) -> torch.Tensor:
        return torch.empty(self.out_bytes, dtype=torch.uint8).pin_memory()

    def unpack_output(self, buf: torch.Tensor):
        d = self.cache.desc
        O = buf[:self.lse_off].view(torch.float32).view(self.cache.O.shape)
        L = buf[self.lse_off:].view(torch.float32).view(self.cache.LSE.shape)
        return O, L

    # ------------------------------------------------------------------ one step
    def step(self, i: int, host_in: torch.Tensor, host_out: torch.Tensor) -> None:
        c, k = self.cache, i & 1
        din, dout = self.dev_in[k], self.dev_out[k]
        with torch.cuda.stream(self.s_in):
            if self.used[k]:
                self.s_in.wait_event(self.ev_comp[k])      # slot k's inputs are no longer read
            din.copy_(host_in, non_blocking=True)
            self.ev_in[k].record(self.s_in)
        q = din[self.q_off:self.q_off + self.q_elems * 2]
        sl = din[self.sl_off:self.sl_off + c.batch * 4]
        tabs = [din[self.tab_off + s * self.tab_elems * 4:self.tab_off + (s + 1) * self.tab_elems * 4]
                for s in range(c.D)]
        o_dev = dout[:self.lse_off]
        l_dev = dout[self.lse_off:]
        self.s_comp.wait_event(self.ev_in[k])
        if self.used[k]:
            self.s_comp.wait_event(self.ev_out[k])         # slot k's results have been read back
        dcp.dcp_decode_partial_all(c.desc, q, c.pools, c.pool_pages, tabs, sl, c.D, list(c.O_parts),
                                   list(c.LSE_parts), c.workspace, stream=self.s_comp)
        dcp.dcp_lse_merge(list(c.O_parts), list(c.LSE_parts), c.D, self.rows,
                          c.desc.head_dim_v, o_dev, l_dev, stream=self.s_comp)
        self.ev_comp[k].record(self.s_comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.ev_comp[k])
            host_out.copy_(dout, non_blocking=True)
            self.ev_out[k].record(self.s_out)
        self.used[k] = True

    def synchronize(self) -> None:
        for st in (self.s_in, self.s_comp, self.s_out):
            st.synchronize()
