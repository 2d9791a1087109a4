"""CPU oracle for the edge-conditioned Clebsch-Gordan tensor-product convolution.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code, tables or constants with the
CUDA library; the two meet only through the seeded inputs of ``workloads``.

What it computes (all fp64, numpy):

* ``so3``     real spherical harmonics of any degree (Cartesian closed form),
              their gradients and Hessians, real-basis so(3) generators and
              the real Clebsch-Gordan tensors obtained as the null space of
              the infinitesimal intertwiner equations.
* ``irreps``  irreps strings and the selection-rule path table.
* ``radial``  the two radial bases and their first two derivatives.
* ``conv``    the operator through the *conventional* schedule named in the
              abstract of "Sobek" (arXiv 2607.18074): per-edge weights
              W_e = sum_k b_ek Theta_k are materialised, per-edge messages are
              formed and scatter-added to receivers; backward and double
              backward are the explicit adjoints of that schedule.  Two
              operator families: "full" (Theta[p] is R x C_in x C_out) and
              "channelwise" (Theta[p] is R x C, W_e[p] diagonal).

Sources: "Sobek: streaming edge-conditioned equivariant tensor-product
convolution" (arXiv 2607.18074), abstract -- the operator (radial projection,
spherical-harmonic coupling, graph aggregation, fully connected multiplicity
mixing) and its three differentiation orders; "The Price of Freedom: Exploring
Expressivity and Runtime Tradeoffs in Equivariant Tensor Products", Approach
and Key results -- the Clebsch-Gordan coupling and its selection rules
(interactability), and the antisymmetric 1o x 1o -> 1e coupling.

Every function is pinned by tests in ``tests/test_oracle_*.py`` against facts
the mathematics fixes (orthogonality, closed forms, equivariance under O(3),
finite differences, brute force, special cases).  Parity unpinned: absolute
output values for the pages' own workloads, which the pages do not print.
"""

from . import irreps, radial, so3, conv  # noqa: F401
