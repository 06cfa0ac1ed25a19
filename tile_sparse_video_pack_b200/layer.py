"""One tile-sparse attention layer: a plan, its device buffers and its score weights."""
from __future__ import annotations

from .vsa import Plan, make_desc, k_from_sparsity


class TileSparseAttention:
    """Runs pack -> score -> select -> sparse attention -> unpack on token-major bf16 Q, K, V.

    ``proj_q`` / ``proj_k``: fp32 CUDA tensors -- the gate G ([d, d], the same
    tensor for both) for mean-pool scoring, or per-head TripPool projections
    ([heads, 3d, p]). ``direct=True`` (plans with ``info.direct_attn``) runs
    pool -> score -> select -> sparse attention straight on the token-major
    tensors and allocates no packed copies: less memory, about three times the
    attention time (see vsa_sparse_attn_direct).
    """

    def __init__(self, plan: Plan, proj_q, proj_k, with_lse: bool = False, device=None, direct: bool = False):
        self.plan = plan
        self.proj_q = proj_q
        self.proj_k = proj_k
        if direct and not plan.info.direct_attn:
            raise ValueError("this plan's tiles are not boxes of the token-major tensors (info.direct_attn == 0)")
        self.direct = direct
        self.bufs = plan.allocate(device, with_lse=with_lse, packed=not direct)

    @classmethod
    def from_config(cls, cfg, sparsity, proj_q, proj_k, k_per_head=None, **kw):
        return cls(Plan.from_config(cfg, sparsity, k_per_head=k_per_head), proj_q, proj_k, **kw)

    def forward(self, q, k, v, out=None, stream=None):
        """Token-major ``[B, N, heads, d]`` bf16 CUDA tensors -> output of the same shape."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        if self.plan.info.n_ref_tiles or self.direct:
            return self.stages(q, k, v, out, stream)   # R2VA budgets, or tiles straight from q, k, v
        self.plan.layer_forward(q, k, v, self.proj_q, self.proj_k, self.bufs, out, stream=stream)
        return out

    __call__ = forward

    def stages(self, q, k, v, out, stream=None):
        """The calls one by one (same result as :meth:`forward`); with reference segments,
        the reference tiles are scored and selected and the attention uses that selection."""
        b, p = self.bufs, self.plan
        if self.direct:
            p.tile_pool(q, k, b["workspace"], stream)
            p.tile_score_pooled(self.proj_q, self.proj_k, b["scores"], b["workspace"], stream)
            p.topk_select(b["scores"], b["idx"], stream)
            p.sparse_attn_direct(q, k, v, b["idx"], out, b["lse"], stream)
            return out
        p.tile_pack_pool(q, k, v, b["qp"], b["kp"], b["vp"], b["workspace"], stream)
        p.tile_score_pooled(self.proj_q, self.proj_k, b["scores"], b["workspace"], stream)
        p.topk_select(b["scores"], b["idx"], stream)
        if p.info.n_ref_tiles:
            p.ref_score(b["kp"], self.proj_k, b["scores_ref"], b["workspace"], stream)
            p.topk_select_ref(b["scores_ref"], b["idx_ref"], stream)
            p.sparse_attn_ref(b["qp"], b["kp"], b["vp"], b["idx"], b["idx_ref"], b["op"], b["lse"], stream)
        else:
            p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], b["lse"], stream)
        p.tile_unpack(b["op"], out, stream)
        return out


__all__ = ["TileSparseAttention", "Plan", "make_desc", "k_from_sparsity"]
