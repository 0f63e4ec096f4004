"""Multi-scale token geometry of a next-scale (VAR) token stack.

[HeatKV] Method step 1 / Figure 1 caption: the model generates token maps of
increasing scale; [Review] Figure 2 caption: the cache grows with each scale;
[Review] Figure 3 caption: tokens of a scale are laid out in raster order.
Scale s is a side_s x side_s map, so it holds n_s = side_s^2 tokens; the
stack stores scales in ascending order, raster order inside a scale.
"""
from __future__ import annotations


class ScaleGeometry:
    """n_s, off_s (first token of scale s), L_k (= off_k + n_k: keys visible to
    scale k under block-causal attention), T (all tokens), and the source
    scale of every token."""

    def __init__(self, sides):
        self.sides = [int(s) for s in sides]
        self.S = len(self.sides)
        self.n = [s * s for s in self.sides]
        self.off = []
        acc = 0
        for n in self.n:
            self.off.append(acc)
            acc += n
        self.T = acc
        self.L = [self.off[k] + self.n[k] for k in range(self.S)]
        self.scale_of = []
        for s in range(self.S):
            self.scale_of.extend([s] * self.n[s])
