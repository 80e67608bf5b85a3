"""FP64 CPU oracle for the NanoQuant hot path (calibration preconditioners + LB-ADMM).

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously-correct
restatement of what the method computes, written from the NanoQuant pages
(arXiv 2602.06694 summaries).  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library (``rank_binary_factorization_b200``) never imports it and shares
no code, table or constant generator with it: the two are independent so that
agreement between them means something.

Modules
-------
``bpw``      bits-per-weight accounting and per-layer rank selection.
``splitmix`` the counter-based generator that draws the initial signs of V.
``calib``    per-channel second/fourth moments and the diagonal Ledoit-Wolf
             shrinkage that yields the preconditioners D_in, D_out.
``lbadmm``   the Latent Binary ADMM iteration, magnitude balancing, scale
             extraction, sign packing and the reconstruction error.
``brute``    exhaustive sign-pattern search on tiny matrices (C, via ctypes).
``gd``       the gradient-descent latent update (a solver variant) and LB-ADMM with it.

Every function names the passage of the pages it follows.  Where the pages are
silent the plainest reading is taken and stated in the function's docstring.
Parity status: every function here is pinned by a ``-m "not gpu"`` test against
something other than itself (closed forms, library routines on special cases,
brute force, published test vectors); none is "parity unpinned".
"""
