"""Independent fp64 CPU oracle for the fused Gaussian-mixture EM step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library under
``ivf_quantizer_b200/`` and its Python binding) may import, call, link or run
anything here.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code, tables or helpers with the CUDA
path; the only thing both sides consume is the seeded input generators in
``synth/``, which hold none of the method's arithmetic.

Source of truth: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
Clustering" (Bloch, Gera, Orbach, Eytan, Toledo; arXiv 2606.10896), §2
(Gaussian mixture, log-likelihood, E-step, M-step Eqs. (1)-(3)) and §4.2-4.3
(argmax and top-2 multi-assignment).  The oracle follows those definitions, not
Algorithm 1's tiled schedule: it materialises the dense responsibility matrix
(row-chunked only to bound RAM), exactly what the fused kernel avoids.

Modules
  gmm_oracle  NumPy fp64 E-step / M-step / loglik / fit / soft-assign.
  brute       pure-Python loops with math.fsum, for tiny inputs only.

Every oracle function is pinned by a ``-m "not gpu"`` test to something other
than itself (closed forms, library special cases, invariants, brute force);
no function is "parity unpinned".
"""
