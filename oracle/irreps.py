"""Irreps strings and the ir_mul feature layout (oracle; test infrastructure).

Sobek §2.2: a feature is a direct sum of blocks x_{l,sigma} in R^{C x (2l+1)},
with total width C_x = sum C (2l+1). Sobek §4.5: kernels use the ir_mul layout,
where adjacent multiplicity channels are contiguous inside each irrep block, so a
block of multiplicity C and degree l occupies (2l+1)*C consecutive scalars laid
out as [m][u] (m = -l..l, u = 0..C-1).
"""
from __future__ import annotations

import re
from dataclasses import dataclass
from typing import List


@dataclass(frozen=True)
class Block:
    mul: int      # multiplicity C (number of channels)
    l: int        # degree
    p: int        # parity, +1 (even, "e") or -1 (odd, "o")
    offset: int   # first scalar of the block in the ir_mul row

    @property
    def dim(self) -> int:
        return 2 * self.l + 1

    @property
    def size(self) -> int:
        return self.mul * self.dim


_TERM = re.compile(r"^\s*(?:(\d+)\s*x\s*)?(\d+)\s*([eo])\s*$")


def parse(s: str) -> List[Block]:
    """Parse '8x0e+8x1o+8x2e' into ir_mul blocks, in the order written."""
    blocks = []
    off = 0
    for term in s.split("+"):
        m = _TERM.match(term)
        if not m:
            raise ValueError(f"bad irreps term {term!r} in {s!r}")
        mul = int(m.group(1)) if m.group(1) else 1
        l = int(m.group(2))
        p = 1 if m.group(3) == "e" else -1
        if mul <= 0:
            raise ValueError(f"multiplicity must be positive in {s!r}")
        b = Block(mul, l, p, off)
        blocks.append(b)
        off += b.size
    return blocks


def dim(blocks: List[Block]) -> int:
    return sum(b.size for b in blocks)


def block_view(row, b: Block):
    """View the scalars of block b in an ir_mul row (or rows) as [..., 2l+1, mul]."""
    seg = row[..., b.offset:b.offset + b.size]
    return seg.reshape(seg.shape[:-1] + (b.dim, b.mul))
