"""The attention layer around the core, for callers that want a module.

discosf.com/news/5175395 §3.1 describes the layer: a value projection, an
output projection, and two linear heads on the query that predict, per head,
level and point, the two offset components and one attention logit; the
offsets start at zero and the logit head with Xavier weights.  Here the
projections and heads are torch linear layers (library GEMMs, outside the
operator's boundary) and everything between them — locations, softmax,
sampling, weighted sum and all their gradients — runs in the fused kernels of
libmsda.so through MSDeformAttnFusedFunction.
"""
from __future__ import annotations

from typing import Optional

import torch
from torch import nn

from .binding import MSDeformAttnFusedFunction


class MSDeformAttn(nn.Module):
    """Multi-scale deformable attention layer.

    forward(query [B, Q, C], reference_points [B, Q, 2] normalized (x, y),
    input_flatten [B, S, C], spatial_shapes [L, 2] int64 (H, W),
    level_start_index [L] int64, padding_mask [B, S] bool or None) -> [B, Q, C].

    One reference point per query, shared by the levels (the fused kernels'
    form).  Padded keys (padding_mask True) get a zero value row.
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
        S = input_flatten.shape[1]
        M, L, K = self.n_heads, self.n_levels, self.n_points
        if reference_points.shape != (B, Q, 2):
            raise ValueError("reference_points must be [B, Q, 2] (one point per query)")
        if spatial_shapes.shape != (L, 2):
            raise ValueError(f"spatial_shapes must be [{L}, 2]")
        value = self.value_proj(input_flatten)
        if padding_mask is not None:
            value = value.masked_fill(padding_mask[..., None], 0.0)
        value = value.reshape(B, S, M, self.d_model // M).contiguous()
        offsets = self.sampling_offsets(query).float().reshape(B, Q, M, L, K, 2).contiguous()
        logits = self.attention_weights(query).float().reshape(B, Q, M, L * K).contiguous()
        out = MSDeformAttnFusedFunction.apply(value, spatial_shapes, level_start_index,
                                              reference_points.float().contiguous(), offsets, logits)
        return self.output_proj(out.reshape(B, Q, self.d_model))
