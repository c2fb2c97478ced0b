"""RecsaLayer: allocates the KV cache and workspace with PyTorch and drives
one recsa_ctx through the C ABI. Marshalling only; the work runs in
librecsa.so."""
from __future__ import annotations

import torch

from . import recsa as _r


class RecsaLayer:
    def __init__(self, batch, n_kv_heads, n_q_heads, head_dim, branching, k, capacity, pooler_w: torch.Tensor,
                 dtype=torch.bfloat16, rope_base=1e6, max_chunk=0, device="cuda", stream=None, page_size=0,
                 num_pages=0, page_table=None):
        """page_size > 0: a paged token cache, a pool of num_pages pages of
        page_size tokens (k_cache, v_cache [num_pages][H_kv][page_size][d])
        with page_table [B][max_pages] (int32; copied to the device)."""
        self.cfg = _r.make_config(batch, n_kv_heads, n_q_heads, head_dim, branching, k, capacity, dtype, rope_base,
                                  max_chunk)
        self.dtype, self.device = dtype, torch.device(device)
        self.page_size = page_size
        if page_size:
            self.k_cache = torch.zeros(num_pages, n_kv_heads, page_size, head_dim, dtype=dtype, device=device)
            self.page_table = torch.as_tensor(page_table, dtype=torch.int32).to(device).contiguous()
        else:
            self.k_cache = torch.zeros(batch, n_kv_heads, capacity, head_dim, dtype=dtype, device=device)
            self.page_table = None
        self.v_cache = torch.zeros_like(self.k_cache)
        self.workspace = torch.zeros(_r.workspace_bytes(self.cfg), dtype=torch.uint8, device=device)
        w = pooler_w.to(device=device, dtype=dtype).contiguous()
        self.w_master = w.float().clone()  # fp32 master copy of the pooler (distillation updates it)
        self.ctx = _r.Context(self.cfg, self.k_cache, self.v_cache, self.workspace, w, stream, self.page_table,
                              page_size)
        torch.cuda.current_stream(self.device).synchronize() if stream is None else stream.synchronize()
        self._scratch = None

    @property
    def G(self) -> int:
        return self.cfg.n_q_heads // self.cfg.n_kv_heads

    def load(self, K: torch.Tensor, V: torch.Tensor, lengths, stream=None):
        """Copy tokens [B][H][L][d] into the cache (through the page table
        when paged) and build the tree over the first lengths[b] tokens of
        each sequence."""
        L = K.shape[2]
        if self.page_size:
            P = self.page_size
            table = self.page_table.cpu()
            for b in range(K.shape[0]):
                for pg in range(-(-L // P)):
                    n = min(P, L - pg * P)
                    dst = int(table[b, pg])
                    self.k_cache[dst, :, :n].copy_(K[b, :, pg * P:pg * P + n], non_blocking=True)
                    self.v_cache[dst, :, :n].copy_(V[b, :, pg * P:pg * P + n], non_blocking=True)
        else:
            self.k_cache[:, :, :L].copy_(K, non_blocking=True)
            self.v_cache[:, :, :L].copy_(V, non_blocking=True)
        self.ctx.build_tree(lengths, stream)

    def load_clustered(self, K: torch.Tensor, V: torch.Tensor, lengths, Z: torch.Tensor, stream=None):
        """LSA-style variant: place tokens [B][H][L][d] into the cache in the
        clustered order of the learned directions Z [J_cap][d] (fp32) and build
        the tree over them. Returns perm [B][H][capacity] (int32, device):
        the source token at each cache position (positions < lengths[b])."""
        if getattr(self, "_cluster_scratch", None) is None:
            self._cluster_scratch = torch.empty(self.ctx.cluster_scratch_bytes(), dtype=torch.uint8,
                                                device=self.device)
        K = K.to(device=self.device, dtype=self.dtype).contiguous()
        V = V.to(device=self.device, dtype=self.dtype).contiguous()
        Z = Z.to(device=self.device, dtype=torch.float32).contiguous()
        perm = torch.full((self.cfg.batch, self.cfg.n_kv_heads, self.cfg.capacity), -1, dtype=torch.int32,
                          device=self.device)
        self.ctx.cluster_load(K, V, lengths, Z, perm, self._cluster_scratch, stream)
        return perm

    def tokens(self, b: int, L: int):
        """Keys and values [H][L][d] of sequence b's first L tokens (read
        back through the page table when paged)."""
        if not self.page_size:
            return self.k_cache[b, :, :L], self.v_cache[b, :, :L]
        P = self.page_size
        pages = [int(x) for x in self.page_table[b, :-(-L // P)].cpu()]
        k = torch.cat([self.k_cache[pg] for pg in pages], dim=1)[:, :L]
        v = torch.cat([self.v_cache[pg] for pg in pages], dim=1)[:, :L]
        return k, v

    def append(self, k_new, v_new, stream=None):
        self.ctx.append(k_new, v_new, stream)

    def decode(self, q, out=None, sel_out=None, rows_out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        self.ctx.decode(q, out, sel_out, rows_out, stream)
        return out

    def append_decode(self, k_new, v_new, q, out=None, sel_out=None, rows_out=None, stream=None):
        """One decode step in one launch: append k_new, v_new [B][1][H_kv][d],
        then attend q [B][H_q][d] over the grown tree."""
        if out is None:
            out = torch.empty_like(q)
        self.ctx.append_decode(k_new, v_new, q, out, sel_out, rows_out, stream)
        return out

    def prefill(self, q, k, v, out=None, sel_out=None, rows_out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        need = self.ctx.prefill_scratch_bytes(q.shape[1])
        if self._scratch is None or self._scratch.numel() < need:
            self._scratch = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        self.ctx.prefill(q, k, v, out, sel_out, self._scratch, rows_out, stream)
        return out

    # ------------------------------------------------------------ gradients

    def zero_grad(self):
        """Allocates (first call) or clears the fp32 gradients: dk, dv shaped
        like the cache, dw [d][d], and the node accumulators."""
        if getattr(self, "dk", None) is None:
            self.dk = torch.zeros(self.k_cache.shape, dtype=torch.float32, device=self.device)
            self.dv = torch.zeros_like(self.dk)
            self.dw = torch.zeros(self.cfg.head_dim, self.cfg.head_dim, dtype=torch.float32, device=self.device)
            self._bwd_scratch = torch.zeros(max(self.ctx.backward_scratch_bytes(), 256), dtype=torch.uint8,
                                            device=self.device)
        else:
            self.dk.zero_()
            self.dv.zero_()
            self.dw.zero_()
            self._bwd_scratch.zero_()

    def decode_backward(self, q, dout, sel, dq=None, stream=None):
        """Gradients of the last decode's output with its selections sel
        [B][H_kv][J_cap][k] held fixed: returns dq [B][H_q][d] (fp32) and adds
        the token entries' gradients into self.dk, self.dv and the summaries'
        into the node accumulators (carried down by tree_backward)."""
        if getattr(self, "dk", None) is None:
            self.zero_grad()
        if dq is None:
            dq = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        self.ctx.decode_backward(q, dout, sel, dq, self.dk, self.dv, self._bwd_scratch, stream)
        return dq

    def tree_backward(self, stream=None):
        """Carries the node accumulators into self.dk, self.dv and self.dw."""
        if getattr(self, "dk", None) is None:
            self.zero_grad()
        self.ctx.tree_backward(self.dk, self.dv, self.dw, self._bwd_scratch, stream)

    def distill_step(self, q, target, lr, dw_out=None, stream=None):
        """One gradient-descent step of the pooler towards dense attention:
        target [B][H_q][d] (fp32) are the dense outputs for q. Returns the
        step's loss (a device scalar); self.w_master holds the new pooler
        and the tree has been rebuilt under it."""
        if getattr(self, "_distill_scratch", None) is None:
            self._distill_scratch = torch.empty(max(self.ctx.distill_scratch_bytes(), 256), dtype=torch.uint8,
                                                device=self.device)
        loss = torch.empty((), dtype=torch.float32, device=self.device)
        self.ctx.distill_step(q, target.contiguous(), lr, self.w_master, self._distill_scratch, loss, dw_out,
                              stream)
        return loss

    def query_stats(self, stream=None):
        return self.ctx.query_stats(stream)

    def lengths(self):
        return self.ctx.lengths()

    def level(self, j):
        return self.ctx.level(j)

    def tree_shape(self):
        return self.ctx.tree_shape()

    def check(self, stream=None):
        self.ctx.check_device(stream)

    def close(self):
        self.ctx.close()
