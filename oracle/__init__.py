"""CPU oracle for the E2Former-V2 on-the-fly equivariant attention layer.

TEST INFRASTRUCTURE ONLY. Plain, slow, fp64 numpy/scipy code that computes
the layer the dense way, so that the CUDA path can be checked against it.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import it. The product path (``atomistic_cell_list_b200``) never
imports, calls or links anything here, and this package never imports the
product path: the only shared code is the seeded input generator module
``workloads``, which holds none of the layer's arithmetic.

Source: "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
Memory" (arXiv 2601.16622), as summarised on the gist.science page,
Technical Summary section 2 (2.1 EAAS with Lemma 4.1 and the re-indexing
rule Eq. 13; 2.2 node-centric factorisation Eq. 6, streaming reduction,
online softmax) and the fugumt abstract page. The pages print no formula;
every reading taken where they are silent is stated in the docstring of the
function that implements it.

Modules:
  sh         real spherical harmonics (closed-form Legendre polynomials)
  cg         complex Clebsch-Gordan (Racah's formula, exact rationals) and
             the real coupling tensors Q
  wigner     real Wigner-D matrices from their definition Y(Rv) = D(R) Y(v)
  eaas       SO(2) weights <-> dense path weights (Lemma 4.1 + Eq. 13)
  layer      radial basis, gates, logits, two-pass softmax, dense messages
  neighbors  the exact fp32 cutoff predicate, brute force and KD-tree search
  grad       the same layer in plain PyTorch fp64, differentiated by autograd
             (gradients for the backward pass)
  sixj       the Wigner-6j node-level convolution variant, edge by edge, and
             Racah's 6j formula (for the pins)
"""
