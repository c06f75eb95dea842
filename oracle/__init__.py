"""CPU oracle for the W4A4 quantized linear layer (test infrastructure).

This package is the plain, slow reference the CUDA path is checked against.
It is test infrastructure only: the product path never imports, links or runs
it. Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it. It shares no code, table
or helper with the CUDA library.

Everything is NumPy in float64 unless a step fixes another precision:

* the block transform (KroQuant commentary, section 02; OrbitQuant commentary,
  section 03, equation RPBH(X) = X P H D) -- ``oracle.transforms``;
* per-token centring and exact rank-1 mean restore (CentriQ summary, abstract)
  -- ``oracle.layer``;
* the SVD low-rank split with a 16-bit branch and a 4-bit residual (SVDQuant
  explainer, section 3) -- ``oracle.layer.prepare``;
* the MXFP4 format the KroQuant commentary (section 03) names, defined by the
  OCP Microscaling Formats v1.0 specification (E2M1 elements, one E8M0 scale
  per 32 elements) -- ``oracle.mxfp4``.

Every function is pinned by ``tests/test_oracle_*.py`` to something other
than itself (closed forms, textbook identities, brute force, hand-derived
fixtures under ``tests/golden/``). Parity unpinned: none of the functions here;
the learned Kronecker factors themselves are synthetic stand-ins (see the
``synthetic`` package), which is a property of the inputs, not of this code.
"""
from . import bf16, mxfp4, transforms, layer  # noqa: F401

__all__ = ["bf16", "mxfp4", "transforms", "layer"]
