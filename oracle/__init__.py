"""CPU oracle for the edge-conditioned Clebsch-Gordan tensor-product convolution.

THIS PACKAGE IS TEST INFRASTRUCTURE. It is a plain, slow, obviously correct fp64
restatement of what the operator computes, written from the method's definition:

* Sobek: Streaming Equivariant Tensor Product Convolutions, §2.2 (irreps and the
  path selection rule), §2.4 (the convolution and the radial factorisation
  W = phi A), §2.5 (the materialised schedule), §3.1-3.2 (reassociation and the
  first backward), §4.2 (receiver-factorised state S and m = S A).
* LunaTP: Enabling Efficient and Scalable Tensor Product for Equivariant MLIPs,
  §2.1 Eq. 1 (component formula of the CG tensor product), Algorithm 1 (standard
  convolution), Appendix F Algorithm 2 (first-order derivatives).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it. The product path (the C-ABI library and its Python
binding) never imports, links or executes anything here, and this package never
imports the product path: the two share no code, tables or constants. The only
code both sides see is the seeded input generator in ``inputs/``, which holds
none of the operator's arithmetic.

Modules
-------
irreps  : irreps strings, ir_mul block layout
cg      : exact complex Clebsch-Gordan coefficients (Racah formula in rational
          arithmetic) and their real-basis form
sh      : real spherical harmonics (component normalisation) and real Wigner-D
paths   : path enumeration, weight layout, N_w, work model
csr     : receiver CSR and its source transpose
conv    : naive materialised forward/backward, and the two reassociated
          schedules (streaming, receiver-factorised) used as brute-force checks

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_*.py``
against something other than itself (closed forms, an independent library,
invariants, values printed on the pages, finite differences).
"""
