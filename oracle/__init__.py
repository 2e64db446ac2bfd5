"""CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
Python binding) imports, calls, links or executes anything in this package.  The
only users are ``tests/``, ``__graft_entry__.smoke()`` (which checks one small GPU
result against it) and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py``.

Two independent implementations live here:

* ``attention.py`` -- NumPy, fp64.  The plain definition of attention written out:
  the full score rows are materialised (a chunk of query rows at a time), an exact
  max-subtracted softmax is taken per row, and the outputs and gradients follow by
  ordinary matrix products.  No online softmax, no tiling over keys.
* ``brute.c`` -- scalar C, fp64 triple loops, one (batch, head) slice at a time;
  used on tiny shapes to check ``attention.py`` against something that shares no
  code with it.

What the pages fix about the computation:

* "Flash Attention spiegata: una guida completa" (datacamp), section
  "Attention standard vs Flash attention": the tiled method is not an
  approximation; its output is mathematically the same as standard
  self-attention.
* "Flash Attention 2: attivarla (llama.cpp, Ollama, vLLM)" (qualellm.it), section
  "Perché Flash Attention 2": the result does not change, only the way it is
  computed -- which is why GPU results are compared within a tolerance.
* "Flash Attention spiegata", section "Ricomputazione": the backward pass
  recomputes the scores instead of storing them.

The formula itself, the scale, the causal mask and the log-sum-exp convention are
not on the pages; they come from the problem statement
O = softmax(Q K^T * scale [+ causal mask]) V and are read as follows (each reading
is the plainest one):

* causal: query row i sees keys 0..i (lower triangle including the diagonal);
* LSE_i: natural log of sum_j exp(S_ij) over the unmasked keys of row i, in
  units of the scaled scores S = scale * Q K^T;
* backward of the loss L with dL/dO = dO: dV = P^T dO, dP = dO V^T,
  D_i = sum_j P_ij dP_ij, dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q;
* sliding window W (causal only): query i sees keys i - W + 1 .. i;
* decode-like attention (``attn_fwd_decode_ref``): the Nq <= Nk queries are the
  last Nq positions, so with the causal mask query i sees keys 0 .. Nk - Nq + i;
* 8-bit inputs (``attn_fwd_fp8_ref``): E4M3 codes (bias 7, three mantissa bits,
  no infinities; ``e4m3_decode`` follows the format's definition) times a
  per-tensor scale, then the plain definition above.

Every function is pinned by ``tests/test_oracle.py`` against things other than
itself: the scalar brute force, PyTorch's fp64 CPU attention and autograd,
closed forms, invariances and central finite differences.
"""

from .attention import (  # noqa: F401
    attn_fwd_decode_ref,
    attn_fwd_fp8_ref,
    e4m3_decode,
    attn_fwd_ref,
    attn_fwd_rows_ref,
    attn_bwd_ref,
    attn_probs_ref,
)
