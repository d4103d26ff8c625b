"""D interleaved paged KV shards on one GPU, driven through the C ABI.

``ShardedPagedCache`` owns the device buffers of one decode problem: the D
shard pools, their block tables, the per-shard partial outputs, the merged
output and the workspace.  torch only allocates memory here; the tables are
built by ``dcp_build_block_table``, the cache write is ``dcp_place_kv``, and a
decode step is ``dcp_decode_partial_all`` (or D ``dcp_decode_partial`` calls)
followed by ``dcp_lse_merge``.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from . import dcp


class ShardedPagedCache:
    def __init__(self, layout: int, num_q_heads: int, num_kv_heads: int, head_dim_qk: int, head_dim_v: int,
                 block_size: int, D: int, seq_lens: Sequence[int], softmax_scale: float, perm_seed: int = 0,
                 device="cuda", pool_fill: Optional[int] = None):
        self.D = D
        self.device = torch.device(device)
        self.seq_lens = [int(x) for x in seq_lens]
        self.batch = len(self.seq_lens)
        mlb, num_pages = dcp.dcp_block_table_extent(self.seq_lens, block_size, D)
        self.max_local_blocks = max(1, mlb)
        self.num_pages = num_pages
        self.tables_host, self.local_len = dcp.dcp_build_block_table(self.seq_lens, block_size, D, perm_seed,
                                                                     self.max_local_blocks)
        self.desc = dcp.make_desc(layout, self.batch, num_q_heads, num_kv_heads, head_dim_qk, head_dim_v,
                                  block_size, self.max_local_blocks, softmax_scale)
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
        self.O_parts = torch.empty((D, self.batch, num_q_heads, head_dim_v), dtype=torch.float32, device=self.device)
        self.LSE_parts = torch.empty((D, self.batch, num_q_heads), dtype=torch.float32, device=self.device)
        self.O = torch.empty((self.batch, num_q_heads, head_dim_v), dtype=torch.float32, device=self.device)
        self.LSE = torch.empty((self.batch, num_q_heads), dtype=torch.float32, device=self.device)

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
        rows = self.batch * self.desc.num_q_heads
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
        per = 2 * d.num_kv_heads * d.head_dim_qk * 2 if d.layout == dcp.DCP_LAYOUT_GQA else d.head_dim_qk * 2
        return int(sum(self.seq_lens)) * per
