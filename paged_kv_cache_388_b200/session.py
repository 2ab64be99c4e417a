"""User-facing wrapper: one layer's paged KV cache resident in device memory.

``PagedKVCache`` owns the K and V block pools and the split-KV workspace and
exposes the three operations of the hot path (``write`` = reshape_and_cache,
``copy_blocks``, ``attend`` = decode), each a single C-ABI call on the current
CUDA stream.  ``step_from_host`` runs one whole decode step from host (pinned)
buffers: copy the step's inputs in, write the new K/V, attend, copy the output
back -- the end-to-end path a serving loop takes every iteration.
"""
from __future__ import annotations

import torch

from . import _lib


class PagedKVCache:
    def __init__(self, num_blocks, num_kv_heads, head_dim, block_size, dtype=torch.bfloat16,
                 device="cuda", k_cache=None, v_cache=None, kv_scales=None):
        """dtype torch.uint8 with kv_scales=(k_scale, v_scale) makes an FP8
        (E4M3) cache: ``write`` quantises, ``attend`` decodes the codes."""
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = k_cache if k_cache is not None else torch.empty(shape, dtype=dtype, device=device)
        self.v_cache = v_cache if v_cache is not None else torch.empty(shape, dtype=dtype, device=device)
        assert tuple(self.k_cache.shape) == shape and tuple(self.v_cache.shape) == shape
        self.num_blocks, self.num_kv_heads, self.head_dim, self.block_size = shape[0], shape[1], shape[3], shape[2]
        self.dtype = self.k_cache.dtype
        self.device = self.k_cache.device
        self.fp8 = self.dtype == torch.uint8
        if self.fp8 and kv_scales is None:
            raise ValueError("an FP8 cache needs kv_scales=(k_scale, v_scale)")
        self.k_scale, self.v_scale = kv_scales if kv_scales is not None else (1.0, 1.0)
        self._ws = torch.empty(0, dtype=torch.uint8, device=self.device)
        self._staging = {}

    # ---- the three device operations --------------------------------------
    def write(self, key, value, slot_mapping):
        if self.fp8:
            _lib.pa_reshape_and_cache_fp8(key, value, self.k_cache, self.v_cache, slot_mapping,
                                          self.k_scale, self.v_scale)
        else:
            _lib.pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slot_mapping)

    def copy_blocks(self, block_mapping):
        if block_mapping.shape[0]:
            _lib.pa_copy_blocks(self.k_cache, self.v_cache, block_mapping)

    def host_pool(self, num_blocks):
        """A (K, V) pair of page-locked host pools of ``num_blocks`` blocks with
        this cache's block shape: the CPU tier that blocks are swapped to."""
        shape = (num_blocks,) + tuple(self.k_cache.shape[1:])
        return (torch.empty(shape, dtype=self.dtype, pin_memory=True),
                torch.empty(shape, dtype=self.dtype, pin_memory=True))

    def swap_out(self, host_k, host_v, block_mapping):
        """Copy device blocks to host blocks: block_mapping int64 [P, 2] of
        (device block, host block), on the device or pinned."""
        if block_mapping.shape[0]:
            _lib.pa_swap_blocks(host_k, host_v, self.k_cache, self.v_cache, block_mapping)

    def swap_in(self, host_k, host_v, block_mapping):
        """Copy host blocks back into device blocks: (host block, device block)."""
        if block_mapping.shape[0]:
            _lib.pa_swap_blocks(self.k_cache, self.v_cache, host_k, host_v, block_mapping)

    def workspace(self, num_seqs, num_heads, max_context_len, kv_split_tokens=0):
        need = _lib.pa_decode_workspace_size(num_seqs, num_heads, self.num_kv_heads, self.head_dim,
                                             self.block_size, max_context_len, kv_split_tokens)
        if self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws if need else None

    def attend(self, q, block_tables, context_lens, scale, out=None, query_start_loc=None,
               max_query_len=1, max_context_len=0, kv_split_tokens=0, staged_blocks=None):
        """Over an FP8 cache, chunked-prefill rows (max_query_len > 1) stage
        their sequences' blocks as 16-bit values: ``staged_blocks`` bounds
        them (``batch.staged_blocks_needed``); when it is None it is counted
        from query_start_loc and context_lens, which copies both to the host."""
        if out is None:
            out = torch.empty_like(q)
        mcl = max_context_len or block_tables.shape[1] * self.block_size
        if self.fp8:
            if kv_split_tokens:
                raise ValueError("an FP8 cache takes the library's split policy (kv_split_tokens=0)")
            if query_start_loc is not None and max_query_len > 1:
                if staged_blocks is None:
                    from .batch import staged_blocks_needed
                    staged_blocks = staged_blocks_needed(query_start_loc.cpu(), context_lens.cpu(),
                                                         self.block_size)
                need = _lib.pa_decode_fp8_rows_workspace_size(
                    block_tables.shape[0], q.shape[1], self.num_kv_heads, self.head_dim,
                    self.block_size, mcl, block_tables.shape[1], max(1, staged_blocks))
                if self._ws.numel() < need:
                    self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
                _lib.pa_decode_fp8(out, q, self.k_cache, self.v_cache, block_tables, context_lens,
                                   scale, self.k_scale, self.v_scale, max_context_len=mcl,
                                   workspace=self._ws, query_start_loc=query_start_loc,
                                   max_query_len=max_query_len, staged_blocks=max(1, staged_blocks))
                return out
            ws = self.workspace(block_tables.shape[0], q.shape[1], mcl)
            _lib.pa_decode_fp8(out, q, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                               self.k_scale, self.v_scale, max_context_len=mcl, workspace=ws)
            return out
        ws = self.workspace(block_tables.shape[0], q.shape[1], mcl, kv_split_tokens)
        _lib.pa_decode(out, q, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                       query_start_loc=query_start_loc, max_query_len=max_query_len,
                       max_context_len=mcl, kv_split_tokens=kv_split_tokens, workspace=ws)
        return out

    def attend_shared_prefix(self, q, block_tables, context_lens, group_start, group_shared_blocks,
                             scale, max_group_size=0, out=None, max_context_len=0,
                             staged_blocks=None):
        """Decode (one query row per sequence) where groups of consecutive
        sequences share the leading blocks of their tables: group j is
        sequences group_start[j] .. group_start[j+1]-1 sharing
        group_shared_blocks[j] blocks (see ``batch.shared_prefix_groups``).
        Same result as ``attend``; the shared blocks are read once per group.
        Over an FP8 cache the shared blocks are staged as 16-bit values:
        ``staged_blocks`` bounds their total (when None it is summed from
        group_shared_blocks, which copies it to the host)."""
        if out is None:
            out = torch.empty_like(q)
        mcl = max_context_len or block_tables.shape[1] * self.block_size
        if self.fp8:
            if staged_blocks is None:
                staged_blocks = int(group_shared_blocks.cpu().clamp(min=0).sum())
            staged_blocks = max(1, int(staged_blocks))
            need = _lib.pa_decode_shared_prefix_fp8_workspace_size(
                block_tables.shape[0], q.shape[1], self.num_kv_heads, self.head_dim,
                self.block_size, mcl, block_tables.shape[1], group_shared_blocks.shape[0],
                staged_blocks)
            if self._ws.numel() < need:
                self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            _lib.pa_decode_shared_prefix_fp8(out, q, self.k_cache, self.v_cache, block_tables,
                                             context_lens, group_start, group_shared_blocks, scale,
                                             self.k_scale, self.v_scale, staged_blocks,
                                             max_group_size=max_group_size, max_context_len=mcl,
                                             workspace=self._ws)
            return out
        need = _lib.pa_decode_shared_prefix_workspace_size(block_tables.shape[0], q.shape[1],
                                                           self.num_kv_heads, self.head_dim,
                                                           self.block_size, mcl)
        if self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        _lib.pa_decode_shared_prefix(out, q, self.k_cache, self.v_cache, block_tables, context_lens,
                                     group_start, group_shared_blocks, scale,
                                     max_group_size=max_group_size, max_context_len=mcl,
                                     workspace=self._ws)
        return out

    # ---- one step from host memory ------------------------------------------
    def _dev_like(self, name, t):
        buf = self._staging.get(name)
        if buf is None or buf.shape != t.shape or buf.dtype != t.dtype:
            buf = torch.empty(t.shape, dtype=t.dtype, device=self.device)
            self._staging[name] = buf
        return buf

    def step_from_host(self, q, key, value, slot_mapping, block_tables, context_lens, out, scale,
                       max_context_len=0, kv_split_tokens=0):
        """All arguments are host tensors (pinned for asynchronous copies);
        ``out`` receives the attention output.  Returns after enqueueing."""
        d = {}
        for name, t in (("q", q), ("key", key), ("value", value), ("slot_mapping", slot_mapping),
                        ("block_tables", block_tables), ("context_lens", context_lens)):
            d[name] = self._dev_like(name, t)
            d[name].copy_(t, non_blocking=True)
        self.write(d["key"], d["value"], d["slot_mapping"])
        o = self._dev_like("out", out)
        self.attend(d["q"], d["block_tables"], d["context_lens"], scale, out=o,
                    max_context_len=max_context_len, kv_split_tokens=kv_split_tokens)
        out.copy_(o, non_blocking=True)
        return out

    def capture_step_from_host(self, q, key, value, slot_mapping, block_tables, context_lens, out,
                               scale, max_context_len=0, warmup=2):
        """Capture ``step_from_host`` on these (pinned) host buffers into a CUDA
        graph and return a callable that replays it: each call copies the
        buffers' current contents in, runs the step and copies ``out`` back.
        The caller refills the host buffers between calls."""
        for _ in range(warmup):  # one-time library setup happens outside capture
            self.step_from_host(q, key, value, slot_mapping, block_tables, context_lens, out,
                                scale, max_context_len=max_context_len)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step_from_host(q, key, value, slot_mapping, block_tables, context_lens, out,
                                scale, max_context_len=max_context_len)
        return g.replay

    def capture_pipelined_steps_from_host(self, steps, block_tables, scale, max_context_len=0,
                                          warmup=2):
        """Capture a run of decode steps fed from page-locked host memory into
        one CUDA graph whose copies overlap the neighbouring steps' kernels.

        ``steps`` is a list of dicts of pinned host tensors, one per step:
        ``q``, ``key``, ``value``, ``slot_mapping``, ``context_lens``,
        ``bt_index`` / ``bt_ids`` (int64 flat indices into ``block_tables``
        and the int32 block ids to store there: the entries appended to the
        tables since the previous step) and ``out`` (receives the attention
        output).  ``block_tables`` is the device-resident table, updated in
        place by every step.

        Step i copies its inputs in on a host-to-device stream while step i-1
        computes, runs reshape_and_cache + decode on the current stream, and
        copies its output back on a device-to-host stream while step i+1
        computes; two device staging sets alternate between the steps.
        Returns a callable that replays the whole run."""
        if not steps:
            raise ValueError("no steps")
        dev = self.device
        names = ("q", "key", "value", "slot_mapping", "context_lens", "bt_index", "bt_ids")
        stage = [{n: torch.empty(steps[0][n].shape, dtype=steps[0][n].dtype, device=dev)
                  for n in names} for _ in range(2)]
        outs = [torch.empty(steps[0]["out"].shape, dtype=steps[0]["out"].dtype, device=dev)
                for _ in range(2)]
        flat_bt = block_tables.view(-1)
        mcl = max_context_len or block_tables.shape[1] * self.block_size
        h2d = torch.cuda.Stream(device=dev)
        d2h = torch.cuda.Stream(device=dev)

        def run():
            main = torch.cuda.current_stream(dev)
            ev_k, ev_out = [], []
            h2d.wait_stream(main)
            d2h.wait_stream(main)
            for i, st in enumerate(steps):
                sb, ob = stage[i % 2], outs[i % 2]
                if i >= 2:  # the staging set's previous user has finished its kernels
                    h2d.wait_event(ev_k[i - 2])
                with torch.cuda.stream(h2d):
                    for n in names:
                        sb[n].copy_(st[n], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(h2d)
                main.wait_event(ev_in)
                if i >= 2:  # its output buffer has been copied out
                    main.wait_event(ev_out[i - 2])
                flat_bt.index_copy_(0, sb["bt_index"], sb["bt_ids"])
                self.write(sb["key"], sb["value"], sb["slot_mapping"])
                self.attend(sb["q"], block_tables, sb["context_lens"], scale, out=ob,
                            max_context_len=mcl)
                ev = torch.cuda.Event()
                ev.record(main)
                ev_k.append(ev)
                d2h.wait_event(ev)
                with torch.cuda.stream(d2h):
                    st["out"].copy_(ob, non_blocking=True)
                eo = torch.cuda.Event()
                eo.record(d2h)
                ev_out.append(eo)
            main.wait_stream(h2d)
            main.wait_stream(d2h)

        for _ in range(warmup):  # one-time library set-up happens outside capture
            run()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        return g.replay

    @staticmethod
    def appended_table_entries(block_tables, context_lens, block_size, new_tokens=1):
        """Flat indices into ``block_tables`` and the ids stored there for the
        blocks that this step's last ``new_tokens`` tokens of each sequence
        opened (a token at offset 0 of a block): what a decode step has to send
        to a device-resident table."""
        import numpy as np
        idx, ids = [], []
        width = block_tables.shape[1]
        for i, L in enumerate(np.asarray(context_lens).tolist()):
            for pos in range(max(0, L - new_tokens), L):
                if pos % block_size == 0:
                    b = pos // block_size
                    idx.append(i * width + b)
                    ids.append(int(block_tables[i, b]))
        return (torch.tensor(idx, dtype=torch.int64), torch.tensor(ids, dtype=torch.int32))

    @staticmethod
    def host_bytes(*tensors) -> int:
        return int(sum(t.numel() * t.element_size() for t in tensors))
