"""CPU oracle for the spacetime-attention hot path.  TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct float64 NumPy (and pure-Python loops for tiny
cases) restating what the pages define:

* ``closed_forms``  - token counts, latent lengths, pair counts, divided-attention
  cost and the FLOP estimator;
* ``reference``     - spacetime patchify, factorised 3D RoPE, full attention and
  the two divided passes (time, space), all in float64;
* ``brute``         - the same definitions as scalar Python loops, for inputs of
  a few hundred elements, used to cross-check ``reference``.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library
and imports nothing from it; the one module both sides use is ``synthetic``
(seeded random inputs, no method arithmetic).

Pins: every function here is checked in ``tests/test_oracle_*.py`` against
something other than itself (numbers printed on the pages, closed forms,
invariants, library routines such as ``torch.nn.functional.conv3d`` and
``scaled_dot_product_attention`` in float64, and brute force).  No function is
"parity unpinned".
"""
from . import closed_forms, reference, brute  # noqa: F401
