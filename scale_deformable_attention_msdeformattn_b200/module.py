"""The attention layer around the core, for callers that want a module.

discosf.com/news/5175395 §3.1 describes the layer: a value projection (W'_m of
the formula, §2.2), an output projection (W_m), and two linear heads on the
query that predict, per head, level and point, the two offset components and
one attention logit; the offsets start at zero and the logit head with Xavier
weights.  cf-1.com/news/4799680 §3.2 turns the head's outputs into sampling
locations (reference + offset / (W_l, H_l)) and attention weights (a softmax
over each head's L*K logits).

On the GPU every step runs in libmsda.so, in the mixed precision the
practical guide recommends (lpnh.cn/news/23513 §4.1: bf16 storage, float32
accumulation):
  value_proj   msda_linear on the tensor cores, bf16 output written directly
               in the core's value layout [B, S, M, D]
  heads        msda_query_head: one tensor-core GEMM for both heads whose
               epilogue forms the sampling locations and the softmax (the
               offsets and logits are never written)
  core         msda_forward (bf16 value and output rows, float32 accumulation)
  output_proj  msda_linear, float32 output
The backward runs msda_backward, msda_query_head_backward (the location and
softmax chain rule), the projections' input gradients through msda_linear
(bf16 gradient rows against the transposed bf16 weights) and their weight
gradients as bf16 library matrix products with float32 accumulation
(torch.matmul).  The parameters stay float32 (master weights); the forward
reads them rounded to bf16.
"""
from __future__ import annotations

from typing import Optional

import torch
from torch import nn

from . import binding


class _LayerFunction(torch.autograd.Function):
    """The layer's forward and backward through the library's kernels."""

    @staticmethod
    def forward(ctx, query, reference_points, input_flatten, w_v, b_v, w_h, b_h, w_o, b_o,
                spatial_shapes, level_start_index, padding_mask, M: int, L: int, K: int):
        B, Q, C = query.shape
        S = input_flatten.shape[1]
        D = C // M
        bf16 = torch.bfloat16
        xb = input_flatten.to(bf16).contiguous()
        qb = query.to(bf16).contiguous()
        wvb, whb, wob = (w.to(bf16).contiguous() for w in (w_v, w_h, w_o))
        ref = reference_points.float().contiguous()
        value = binding.linear(xb.view(B * S, C), wvb, b_v.float().contiguous(),
                               out_dtype=bf16).view(B, S, M, D)
        if padding_mask is not None:
            value = value.masked_fill(padding_mask[:, :, None, None], 0.0)
        loc, attn = binding.query_head(qb, whb, b_h.float().contiguous(), ref, spatial_shapes, M, K)
        core = binding.forward(value, spatial_shapes, level_start_index, loc, attn)
        y = binding.linear(core.view(B * Q, C), wob, b_o.float().contiguous(), out_dtype=torch.float32)
        ctx.save_for_backward(xb, qb, wvb, whb, wob, value, loc, attn, core, spatial_shapes,
                              level_start_index,
                              padding_mask if padding_mask is not None else torch.empty(0))
        ctx.dims = (B, Q, S, C, M, L, K)
        ctx.has_mask = padding_mask is not None
        return y.view(B, Q, C).to(query.dtype)

    @staticmethod
    def backward(ctx, grad_y):
        (xb, qb, wvb, whb, wob, value, loc, attn, core, shapes, starts, mask) = ctx.saved_tensors
        B, Q, S, C, M, L, K = ctx.dims
        P = M * L * K
        bf16 = torch.bfloat16
        # the layer's gradients in bf16 as its operands (float32 accumulation):
        # input gradients on the tensor cores through msda_linear with the
        # transposed weights, weight gradients as library GEMMs
        gyb = grad_y.to(bf16).reshape(B * Q, C).contiguous()
        # output projection y = core W_o^T + b_o; the core's grad_output rows
        # are stored in the value dtype (bf16)
        g_core = binding.linear(gyb, wob.t().contiguous(), out_dtype=bf16)
        g_wo = (gyb.t() @ core.view(B * Q, C)).float()
        g_bo = grad_y.float().sum((0, 1))
        gv, gl, ga = binding.backward(value, shapes, starts, loc, attn, g_core.view(B, Q, M, C // M))
        if ctx.has_mask:
            gv = gv.masked_fill(mask[:, :, None, None], 0.0)
        # value projection value = x W_v^T + b_v
        gvb = gv.view(B * S, C).to(bf16)
        g_x = binding.linear(gvb, wvb.t().contiguous(), out_dtype=torch.float32)
        g_wv = (gvb.t() @ xb.view(B * S, C)).float()
        g_bv = gv.view(B * S, C).sum(0)
        # the heads: location / softmax chain rule, then the linear layer
        gh, gref = binding.query_head_backward(attn, gl, ga, shapes,
                                               want_grad_reference_points=ctx.needs_input_grad[1])
        ghb = gh.view(B * Q, 3 * P).to(bf16)
        g_q = binding.linear(ghb, whb.t().contiguous(), out_dtype=torch.float32)
        g_wh = (ghb.t() @ qb.view(B * Q, C)).float()
        g_bh = gh.view(B * Q, 3 * P).sum(0)
        return (g_q.view(B, Q, C), gref, g_x.view(B, S, C), g_wv, g_bv, g_wh, g_bh, g_wo, g_bo,
                None, None, None, None, None, None)


class MSDeformAttn(nn.Module):
    """Multi-scale deformable attention layer.

    forward(query [B, Q, C], reference_points [B, Q, 2] normalized (x, y),
    input_flatten [B, S, C], spatial_shapes [L, 2] int64 (H, W),
    level_start_index [L] int64, padding_mask [B, S] bool or None) -> [B, Q, C]
    (float32, or the query's dtype).

    One reference point per query, shared by the levels.  Padded keys
    (padding_mask True) get a zero value row.  Sizes the kernels need:
    C = M * D with D in {8, 16, 32, 64, 128, 256} and C a multiple of 8;
    L * K a power of two of at most 32; M * L * K a multiple of 32.
    """

    def __init__(self, d_model: int = 256, n_levels: int = 4, n_heads: int = 8, n_points: int = 4):
        super().__init__()
        if d_model % n_heads:
            raise ValueError("d_model must be a multiple of n_heads")
        self.d_model, self.n_levels, self.n_heads, self.n_points = d_model, n_levels, n_heads, n_points
        self.sampling_offsets = nn.Linear(d_model, n_heads * n_levels * n_points * 2)
        self.attention_weights = nn.Linear(d_model, n_heads * n_levels * n_points)
        self.value_proj = nn.Linear(d_model, d_model)
        self.output_proj = nn.Linear(d_model, d_model)
        self.reset_parameters()

    def reset_parameters(self) -> None:
        # zero offsets at start (every point samples its reference point);
        # Xavier for the logit head and the projections, zero biases
        nn.init.zeros_(self.sampling_offsets.weight)
        nn.init.zeros_(self.sampling_offsets.bias)
        for lin in (self.attention_weights, self.value_proj, self.output_proj):
            nn.init.xavier_uniform_(lin.weight)
            nn.init.zeros_(lin.bias)

    def forward(self, query: torch.Tensor, reference_points: torch.Tensor,
                input_flatten: torch.Tensor, spatial_shapes: torch.Tensor,
                level_start_index: torch.Tensor,
                padding_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
        B, Q, _ = query.shape
        M, L, K = self.n_heads, self.n_levels, self.n_points
        if reference_points.shape != (B, Q, 2):
            raise ValueError("reference_points must be [B, Q, 2] (one point per query)")
        if spatial_shapes.shape != (L, 2):
            raise ValueError(f"spatial_shapes must be [{L}, 2]")
        # one head GEMM: offset rows (M, L, K, 2) then logit rows (M, L*K)
        w_h = torch.cat([self.sampling_offsets.weight, self.attention_weights.weight], 0)
        b_h = torch.cat([self.sampling_offsets.bias, self.attention_weights.bias], 0)
        return _LayerFunction.apply(query, reference_points, input_flatten, self.value_proj.weight,
                                    self.value_proj.bias, w_h, b_h, self.output_proj.weight,
                                    self.output_proj.bias, spatial_shapes, level_start_index,
                                    padding_mask, M, L, K)
