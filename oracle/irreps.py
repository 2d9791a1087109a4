"""Irreps strings and the selection-rule path table (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

An irreps string such as ``"64x0e+64x1o"`` lists blocks mul x (l, parity).
A feature vector stores the blocks in string order; inside a block the layout
is [mul][2l+1] with m fastest.

A path (i1, l2, i3) couples input block i1 (degree l1, parity p1) with the
spherical harmonic of degree l2 (parity (-1)^l2) into output block i3 (degree
l3, parity p3).  It exists when |l1 - l2| <= l3 <= l1 + l2 and
p1 * (-1)^l2 == p3 -- the selection rules ("interactability") of "The Price of
Freedom", Approach.  Paths are ordered by output block, then input block, then
l2.  Theta holds one [R][C_in][C_out] block per path, in path order.
"""

from __future__ import annotations

import re
from dataclasses import dataclass


@dataclass(frozen=True)
class Block:
    mul: int
    l: int
    p: int  # +1 even, -1 odd

    @property
    def dim(self) -> int:
        return self.mul * (2 * self.l + 1)


def parse(s: str) -> list[Block]:
    blocks = []
    for tok in s.replace(" ", "").split("+"):
        m = re.fullmatch(r"(\d+)x(\d+)([eo])", tok)
        if not m:
            raise ValueError(f"bad irreps token {tok!r}")
        blocks.append(Block(int(m.group(1)), int(m.group(2)), 1 if m.group(3) == "e" else -1))
    return blocks


def offsets(blocks: list[Block]) -> list[int]:
    out, o = [], 0
    for b in blocks:
        out.append(o)
        o += b.dim
    return out


def dim(blocks: list[Block]) -> int:
    return sum(b.dim for b in blocks)


@dataclass(frozen=True)
class Path:
    i1: int
    l2: int
    i3: int
    l1: int
    l3: int
    c_in: int
    c_out: int
    in_off: int
    out_off: int
    theta_off: int


def paths(irreps_in: str, l_sh_max: int, irreps_out: str, R: int, family: str = "full") -> list[Path]:
    """Paths in canonical order (output block, input block, l2) with their Theta offsets.

    family "full": Theta[p] is R x C_in x C_out (every input channel mixes into every output
    channel); "channelwise": Theta[p] is R x C, one weight per radial function and channel,
    which needs C_in = C_out on every path."""
    if family not in ("full", "channelwise"):
        raise ValueError(f"unknown operator family {family!r}")
    bin_, bout = parse(irreps_in), parse(irreps_out)
    oin, oout = offsets(bin_), offsets(bout)
    out, toff = [], 0
    for i3, b3 in enumerate(bout):
        for i1, b1 in enumerate(bin_):
            for l2 in range(l_sh_max + 1):
                if not (abs(b1.l - l2) <= b3.l <= b1.l + l2):
                    continue
                if b1.p * (-1) ** l2 != b3.p:
                    continue
                if family == "channelwise" and b1.mul != b3.mul:
                    raise ValueError("the channel-wise product needs equal input and output multiplicities")
                out.append(Path(i1, l2, i3, b1.l, b3.l, b1.mul, b3.mul, oin[i1], oout[i3], toff))
                toff += R * b1.mul * (b3.mul if family == "full" else 1)
    return out


def theta_numel(ps: list[Path], R: int, family: str = "full") -> int:
    return sum(R * p.c_in * (p.c_out if family == "full" else 1) for p in ps)
