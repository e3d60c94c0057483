"""A block of interleaved local/global attention layers driven through the C ABI.

The layer schedule and the share map come from ``gemma_layer_schedule``; a
shared layer's cache descriptor is bound to its source with
``gemma_kv_share_bind`` (pointer aliasing, no copy) and its calls carry
``GEMMA_F_SHARED`` so that it neither rotates nor writes K/V. Device memory
(caches, workspace, outputs) is torch-owned; all compute is in the library.
"""
from __future__ import annotations

import torch

from . import native
from .workloads import LayerType, Workload


class AttentionStack:
    def __init__(self, w: Workload, device="cuda", global_capacity: int | None = None,
                 alloc_caches: bool = True):
        self.w = w
        self.device = torch.device(device)
        if w.fixed_kinds:
            self.is_global = [k == "global" for k in w.fixed_kinds]
            self.share_src = list(range(len(w.fixed_kinds)))
        else:
            self.is_global, self.share_src = native.gemma_layer_schedule(w.n_layers, w.ratio, w.n_shared)
        self.n_layers = len(self.is_global)
        if global_capacity is None:
            global_capacity = (w.prior + w.seq) if w.kind == "prefill" else w.len_hi
        self.global_capacity = global_capacity
        self.descs: list[native.gemma_kv_desc] = []
        self.k_cache: list[torch.Tensor] = []
        self.v_cache: list[torch.Tensor] = []
        for l in range(self.n_layers):
            t = self.layer_type(l)
            cap = t.window if t.window > 0 else global_capacity
            d = native.gemma_kv_desc()
            d.layer, d.cache_cap, d.window = l, cap, t.window
            d.n_kv_heads, d.head_dim = t.n_kv_heads, t.head_dim
            d.rope_frac, d.rope_theta, d.shared_from = t.rope_frac, t.rope_theta, -1
            d.k_eq_v = int(self.keqv(l))
            d.kv_int8 = int(w.kv_int8)
            src = self.share_src[l]
            if src >= 0 and src != l:
                native.gemma_kv_share_bind(d, self.descs[src])
                self.k_cache.append(self.k_cache[d.shared_from])
                self.v_cache.append(self.v_cache[d.shared_from])
            else:
                shape = (w.batch, t.n_kv_heads, cap, t.head_dim)
                if alloc_caches:
                    if w.kv_int8:
                        def new_cache():
                            return native.Int8KVCache(*shape, self.device)
                    else:
                        def new_cache():
                            return torch.empty(shape, dtype=torch.bfloat16, device=self.device)
                    kc = new_cache()
                    # K = V: the key cache is the only cache
                    vc = kc if d.k_eq_v else new_cache()
                    d.k_cache, d.v_cache = kc.data_ptr(), (0 if d.k_eq_v else vc.data_ptr())
                else:
                    kc = vc = None
                self.k_cache.append(kc)
                self.v_cache.append(vc)
            self.descs.append(d)

    def layer_type(self, l: int) -> LayerType:
        return self.w.global_ if self.is_global[l] else self.w.local

    def keqv(self, l: int) -> bool:
        """Global layers of a K = V workload read their values from the key cache."""
        return bool(self.w.k_eq_v and self.is_global[l])

    def is_shared(self, l: int) -> bool:
        return self.descs[l].shared_from >= 0

    def owned_cache_bytes(self) -> int:
        seen, total = set(), 0
        for l in range(self.n_layers):
            kc = self.k_cache[l]
            if kc is None or kc.data_ptr() in seen:
                continue
            seen.add(kc.data_ptr())
            per = kc.numel() * (1 if isinstance(kc, native.Int8KVCache) else kc.element_size())
            total += (1 if self.keqv(l) else 2) * per
        return total

    # ------------------------------------------------------------------ prefill
    def prefill_workspace_bytes(self, after_cached: bool | None = None) -> int:
        """Workspace for one prefill layer call; after_cached (default: the
        workload has cached tokens) sizes it for chunks after cached tokens."""
        w = self.w
        if after_cached is None:
            # int8 caches: a shared layer's prefill reads cached rows too
            after_cached = w.prior > 0 or (w.kv_int8 and any(self.is_shared(l) for l in range(self.n_layers)))
        flags = native.GEMMA_F_KV_INT8 if w.kv_int8 else 0
        sizes = []
        for l in range(self.n_layers):
            t = self.layer_type(l)
            if after_cached:
                cap = t.window if t.window > 0 else self.global_capacity
                sizes.append(native.gemma_attn_prefill_workspace_size_cached(
                    w.batch, w.seq, w.n_q_heads, t.n_kv_heads, t.head_dim, t.window, cap, flags))
            else:
                sizes.append(native.gemma_attn_prefill_workspace_size(
                    w.batch, w.seq, w.n_q_heads, t.n_kv_heads, t.head_dim, t.window))
        return max(sizes)

    # ---------------------------------------------- windows of shared local layers
    def _has_sharers(self, l: int) -> bool:
        return any(self.descs[m].shared_from == l for m in range(self.n_layers))

    def _window_source(self, l: int, chunked: bool):
        """For a local layer's chunk after cached tokens on a stack whose
        local layers share K/V: the source layer whose call leaves the K/V
        window in its own workspace (GEMMA_F_SOURCE_WINDOW), else None."""
        if not chunked or self.layer_type(l).window == 0:
            return None
        if self.is_shared(l):
            return self.descs[l].shared_from
        return l if self._has_sharers(l) else None

    def _window_workspace(self, src: int, nbytes: int):
        """The workspace a source layer and its sharers use for one chunk
        (kept per source: layers in between must not write it)."""
        if not hasattr(self, "_win_ws"):
            self._win_ws = {}
        buf = self._win_ws.get(src)
        if buf is None or buf.numel() < nbytes:
            buf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=self.device)
            self._win_ws[src] = buf
        return buf

    def prefill_layer(self, l: int, q, k, v, out, *, workspace, seq_lens_before=None, lse=None,
                      stream=None):
        """One layer's chunk. A local layer after cached tokens whose K/V
        are shared runs, with its sharers, on a workspace of its own."""
        t = self.layer_type(l)
        shared = self.is_shared(l)
        keqv = self.keqv(l)
        flags = (native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0)
        src = self._window_source(l, seq_lens_before is not None)
        if src is not None:
            flags |= native.GEMMA_F_SOURCE_WINDOW
            n = native.gemma_attn_prefill_workspace_size_cached(
                q.shape[0], q.shape[1], q.shape[2], t.n_kv_heads, t.head_dim, t.window, t.window,
                native.GEMMA_F_KV_INT8 if self.w.kv_int8 else 0)
            workspace = self._window_workspace(src, n)
        native.gemma_attn_prefill(
            q, None if shared else k, None if (shared or keqv) else v, self.k_cache[l],
            None if keqv else self.v_cache[l],
            window=t.window, rope_frac=t.rope_frac, rope_theta=t.rope_theta, scale=t.scale,
            out=out, seq_lens_before=seq_lens_before, lse=lse, workspace=workspace, flags=flags,
            stream=stream)

    def prefill_from_host(self, host_in, host_out, dev_bufs, *, workspace, seq_lens_before=None):
        """One prefill pass of every layer on inputs in pinned host memory.

        host_in[l] = (q, k, v) pinned host tensors; host_out[l] a pinned host
        tensor for layer l's output; dev_bufs[l] = (q, k, v, out) device
        buffers of the same shapes. The host->device copies of layer l+1's
        inputs and the device->host copy of layer l-1's output run on their
        own streams while layer l computes, so the two copy directions and
        the attention overlap. Work is ordered after everything already on
        the current stream, and the current stream waits for the last
        output copy: synchronising the current stream covers the whole pass.
        """
        comp = torch.cuda.current_stream(self.device)
        if not hasattr(self, "_copy_streams"):
            self._copy_streams = (torch.cuda.Stream(self.device), torch.cuda.Stream(self.device))
        s_in, s_out = self._copy_streams
        s_in.wait_stream(comp)   # earlier computes are done with the input buffers
        s_out.wait_stream(comp)
        ready = []
        with torch.cuda.stream(s_in):
            for (hq, hk, hv), (q, k, v, _) in zip(host_in, dev_bufs):
                q.copy_(hq, non_blocking=True)
                k.copy_(hk, non_blocking=True)
                v.copy_(hv, non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                ready.append(e)
        for l, (q, k, v, out) in enumerate(dev_bufs):
            comp.wait_event(ready[l])
            self.prefill_layer(l, q, k, v, out, workspace=workspace, seq_lens_before=seq_lens_before,
                               stream=comp)
            done = torch.cuda.Event()
            done.record(comp)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                host_out[l].copy_(out, non_blocking=True)
        comp.wait_stream(s_out)

    # ------------------------------------------------------------------ decode
    def decode_workspace_bytes(self, max_seq_len: int) -> int:
        w = self.w
        return max(native.gemma_attn_decode_workspace_size(
            w.batch, w.n_q_heads, self.layer_type(l).n_kv_heads, self.layer_type(l).head_dim,
            self.layer_type(l).window, max_seq_len) for l in range(self.n_layers))

    def decode_layer(self, l: int, q, k, v, out, *, seq_lens, max_seq_len, workspace, stream=None):
        t = self.layer_type(l)
        shared = self.is_shared(l)
        keqv = self.keqv(l)
        native.gemma_attn_decode(
            q, None if shared else k, None if (shared or keqv) else v, self.k_cache[l],
            None if keqv else self.v_cache[l],
            seq_lens=seq_lens, max_seq_len=max_seq_len, window=t.window, rope_frac=t.rope_frac,
            rope_theta=t.rope_theta, scale=t.scale, out=out, workspace=workspace,
            flags=(native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0),
            stream=stream)

    # ------------------------------------------------------- multi-token decode
    def decode_multi_workspace_bytes(self, tokens: int, max_seq_len: int) -> int:
        w = self.w
        flags = native.GEMMA_F_KV_INT8 if w.kv_int8 else 0
        sizes = []
        for l in range(self.n_layers):
            t = self.layer_type(l)
            cap = t.window if t.window > 0 else self.global_capacity
            sizes.append(native.gemma_attn_decode_multi_workspace_size(
                w.batch, tokens, w.n_q_heads, t.n_kv_heads, t.head_dim, t.window, max_seq_len, cap, flags))
        return max(sizes)

    def decode_multi_layer(self, l: int, q, k, v, out, *, seq_lens, max_seq_len, workspace, stream=None):
        """tokens = q.shape[1] new tokens per sequence (a drafter's proposals
        being checked); seq_lens counts them. Local layers whose K/V are
        shared run, with their sharers, as a chunk after the cached tokens
        on a workspace of their own (GEMMA_F_SOURCE_WINDOW)."""
        t = self.layer_type(l)
        shared = self.is_shared(l)
        keqv = self.keqv(l)
        flags = (native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0)
        src = self._window_source(l, True)
        if src is not None:
            flags |= native.GEMMA_F_SOURCE_WINDOW
            n = native.gemma_attn_decode_multi_workspace_size(
                q.shape[0], q.shape[1], q.shape[2], t.n_kv_heads, t.head_dim, t.window, max_seq_len, t.window,
                flags | (native.GEMMA_F_KV_INT8 if self.w.kv_int8 else 0))
            workspace = self._window_workspace(src, n)
        native.gemma_attn_decode_multi(
            q, None if shared else k, None if (shared or keqv) else v, self.k_cache[l],
            None if keqv else self.v_cache[l],
            seq_lens=seq_lens, max_seq_len=max_seq_len, window=t.window, rope_frac=t.rope_frac,
            rope_theta=t.rope_theta, scale=t.scale, out=out, workspace=workspace, flags=flags,
            stream=stream)
