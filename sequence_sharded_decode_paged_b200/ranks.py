"""Decode context parallelism across D GPUs: one shard per rank.

The pages' multi-GPU method ("Efficient Decode Context Parallelism with vLLM
for Long Context Workloads", A2 方法细节): the KV cache of every request is cut
along the sequence over the D ranks of the DCP group; per decode step each
rank (1) has the full query, (2) attends it against its own KV slice, giving a
partial O_i and LSE_i, and (3) the ranks exchange the partials so that each
ends with the merged output of its own slice of query heads (the pages'
AllGather of (O_i, LSE_i) followed by a ReduceScatter).

Data plane here, per step and rank r (shard r of D, heads r*Hk .. r*Hk + Hk - 1,
Hk = Hq / D):

* ``dcp_decode_partial_owner_major`` (one CUDA kernel launch) writes shard r's
  partial straight into the send buffer in owner order: chunk k holds the O
  rows, then the LSE rows, of the heads rank k owns.
* ``exchange`` is one ``all_to_all_single`` of equal chunks (NCCL over
  NVLink / NVSwitch on B200; gloo on CPU in the tests): rank r sends chunk k to
  rank k and receives, from every rank j, shard j's partial for its own heads.
  Each rank moves (D - 1) / D of one partial -- B * q_len * Hq * (d_v + 1) * 4
  bytes -- in each direction, independent of the context length.
* ``dcp_lse_merge`` (one launch) merges the D received chunks into the merged
  O and LSE of the rank's heads.

With ``exchange="p2p"`` the first two steps are one: every rank maps every
other rank's receive buffer into its address space (CUDA IPC, plain device
memory, no multicast) and ``dcp_decode_partial_to_owners`` stores each owner's
rows straight into that owner's buffer from the decode kernel's epilogue, so
the transfer runs while the partial is still being finished.  The stream's
completion and a barrier of the group then order those stores before the
merge; two receive buffers alternate between steps, so that a rank writing
step t+1's rows never touches a buffer an owner may still be merging.

The query is an input of the step: the pages' AllGather-Q is the caller's
(on one node every rank usually computes the same q already).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from . import dcp


def owner_chunk_floats(batch: int, q_len: int, num_q_heads: int, head_dim_v: int, n_owners: int) -> int:
    """Floats of one owner's chunk: its O rows, then its LSE rows padded to 64 floats
    (the layout ``dcp_decode_partial_owner_major`` writes; ``dcp_owner_chunk_floats``)."""
    rows = batch * q_len * (num_q_heads // n_owners)
    return rows * head_dim_v + (rows + 63) // 64 * 64


def exchange(send: torch.Tensor, recv: torch.Tensor, group=None) -> None:
    """All-to-all of equal chunks: rank r's chunk k lands as chunk r of rank k's ``recv``.

    ``send`` and ``recv`` are flat fp32 tensors of world_size equal chunks, on the device the
    process group's backend serves (CUDA for NCCL, CPU for gloo)."""
    import torch.distributed as dist
    dist.all_to_all_single(recv, send, group=group)


def split_chunks(buf: torch.Tensor, D: int, rows: int, head_dim_v: int):
    """Views of the D chunks of an owner-major buffer: ([O parts], [LSE parts])."""
    chunk = buf.numel() // D
    Os, Ls = [], []
    for k in range(D):
        c = buf[k * chunk:(k + 1) * chunk]
        Os.append(c[:rows * head_dim_v].view(rows, head_dim_v))
        Ls.append(c[rows * head_dim_v:rows * head_dim_v + rows])
    return Os, Ls


def owner_chunk_addresses(recv_bases, rank: int, chunk_floats: int, parity: int):
    """Where rank ``rank``'s decode kernel stores each owner's rows in the folded exchange.

    ``recv_bases[r]`` is the address (in this process) of rank r's pair of receive buffers, each
    D chunks of ``chunk_floats`` fp32; step parity ``parity`` uses buffer 0 or 1.  Owner r takes
    this shard's rows as chunk ``rank`` of its buffer, so after the step owner r's buffer holds
    every shard's rows for its heads in shard order -- the layout ``split_chunks`` reads."""
    D = len(recv_bases)
    return [recv_bases[r] + ((parity * D + rank) * chunk_floats) * 4 for r in range(D)]


class RankShardedDecode:
    """Shard ``rank`` of a D-rank DCP group (D = the group's size) on this process's GPU.

    Holds that shard's pool and block table only; ``place`` writes this shard's tokens of the
    unsharded KV, ``step`` runs one decode step (partial, exchange, merge) and returns the merged
    ``(O, LSE)`` of this rank's heads: ``O[batch][q_len][Hk][d_v]``, ``LSE[batch][q_len][Hk]``.
    ``kv_dtype`` / ``k_scale`` / ``v_scale`` select an FP8 E4M3 pool as in ``dcp_attn_desc``.
    """

    def __init__(self, layout: int, num_q_heads: int, num_kv_heads: int, head_dim_qk: int, head_dim_v: int,
                 block_size: int, seq_lens: Sequence[int], softmax_scale: float, group=None, device="cuda",
                 q_len: int = 1, perm_seed: int = 0, kv_dtype: int = 0, k_scale: float = 1.0,
                 v_scale: float = 1.0, exchange: str = "nccl"):
        import torch.distributed as dist
        if exchange not in ("nccl", "p2p"):
            raise ValueError("exchange must be 'nccl' (all-to-all) or 'p2p' (stores into the owners' buffers)")
        self.exchange_kind = exchange
        self.group = group
        self.rank = dist.get_rank(group)
        self.D = dist.get_world_size(group)
        if num_q_heads % self.D != 0:
            raise ValueError("the query heads must split evenly over the ranks")
        self.device = torch.device(device)
        self.seq_lens = [int(x) for x in seq_lens]
        self.batch, self.q_len = len(self.seq_lens), q_len
        self.Hk = num_q_heads // self.D
        mlb, num_pages = dcp.dcp_block_table_extent(self.seq_lens, block_size, self.D)
        self.max_local_blocks = max(1, mlb)
        tables, self.local_len = dcp.dcp_build_block_table(self.seq_lens, block_size, self.D, perm_seed,
                                                           self.max_local_blocks)
        self.desc = dcp.make_desc(layout, self.batch, num_q_heads, num_kv_heads, head_dim_qk, head_dim_v,
                                  block_size, self.max_local_blocks, softmax_scale, q_len, kv_dtype, k_scale,
                                  v_scale)
        page_bytes = dcp.dcp_kv_page_bytes(self.desc)
        if page_bytes == 0:
            raise ValueError("unsupported attention shape")
        self.pool_pages = int(num_pages[self.rank])
        self.pool = torch.empty(max(1, self.pool_pages) * page_bytes // 2, dtype=torch.int16, device=self.device)
        self.table = torch.from_numpy(np.ascontiguousarray(tables[self.rank])).to(self.device)
        self.seq_lens_dev = torch.tensor(self.seq_lens, dtype=torch.int32, device=self.device)
        self.workspace = torch.empty(dcp.dcp_decode_workspace_bytes(self.desc, self.D), dtype=torch.uint8,
                                     device=self.device)
        dcp.dcp_workspace_init(self.workspace)
        self.chunk = dcp.dcp_owner_chunk_floats(self.desc, self.D)
        self.rows = self.batch * q_len * self.Hk
        self._mapped = []
        if exchange == "nccl":
            self.send = torch.empty(self.D * self.chunk, dtype=torch.float32, device=self.device)
            self.recv = torch.empty_like(self.send)
        else:
            # two receive buffers in one allocation; every rank learns where every other rank's are
            self.recv_pair = torch.empty(2 * self.D * self.chunk, dtype=torch.float32, device=self.device)
            handle, offset = dcp.dcp_ipc_export(self.recv_pair)
            peers = [None] * self.D
            dist.all_gather_object(peers, (self.rank, handle, offset), group=group)
            base_of = {}
            for r, h, off in peers:
                if r == self.rank:
                    base_of[r] = self.recv_pair.data_ptr()
                else:
                    mapped = dcp.dcp_ipc_open(h)
                    self._mapped.append(mapped)
                    base_of[r] = mapped + off
            bases = [base_of[r] for r in range(self.D)]
            self.owner_ptrs = [owner_chunk_addresses(bases, self.rank, self.chunk, i) for i in range(2)]
            self.steps_done = 0
        self.O = torch.empty((self.batch, q_len, self.Hk, head_dim_v), dtype=torch.float32, device=self.device)
        self.LSE = torch.empty((self.batch, q_len, self.Hk), dtype=torch.float32, device=self.device)

    def place(self, kv_src: torch.Tensor, cu_seqlens: torch.Tensor) -> None:
        """Write this shard's tokens of the unsharded KV rows (requests concatenated, as for
        ``dcp_place_kv``); the other shards' rows are skipped (their pools have no pages here)."""
        pools = [None] * self.D
        pages = [0] * self.D
        tables = [self.table] * self.D
        pools[self.rank], pages[self.rank] = self.pool, self.pool_pages
        dcp.dcp_place_kv(self.desc, self.D, kv_src, cu_seqlens, self.seq_lens_dev, tables, pools, pages)

    def step(self, q: torch.Tensor, stream=None):
        """One decode step for the full query ``q`` (``[batch][q_len][Hq][d_qk]`` bf16 bits)."""
        d = self.desc
        if self.exchange_kind == "nccl":
            dcp.dcp_decode_partial_owner_major(d, q, self.pool, self.pool_pages, self.table, self.seq_lens_dev,
                                               self.rank, self.D, self.D, self.send, self.workspace, stream=stream)
            exchange(self.send, self.recv, self.group)
            recv = self.recv
        else:
            import torch.distributed as dist
            i = self.steps_done & 1
            self.steps_done += 1
            dcp.dcp_decode_partial_to_owners(d, q, self.pool, self.pool_pages, self.table, self.seq_lens_dev,
                                             self.rank, self.D, self.owner_ptrs[i], self.workspace, stream=stream)
            # every rank's stores into this rank's chunks are complete before the merge reads them
            (torch.cuda.current_stream(self.device) if stream is None else stream).synchronize()
            dist.barrier(group=self.group)
            recv = self.recv_pair[i * self.D * self.chunk:(i + 1) * self.D * self.chunk]
        Os, Ls = split_chunks(recv, self.D, self.rows, d.head_dim_v)
        dcp.dcp_lse_merge(Os, Ls, self.D, self.rows, d.head_dim_v, self.O, self.LSE, stream=stream)
        return self.O, self.LSE

    def device_error(self) -> int:
        return dcp.dcp_read_device_error(self.workspace)

    def close(self) -> None:
        """Unmap the other ranks' receive buffers (p2p exchange); call on every rank before any of
        them frees its own, e.g. followed by a barrier of the group."""
        for base in self._mapped:
            dcp.dcp_ipc_close(base)
        self._mapped = []
