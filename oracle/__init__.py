"""CPU oracle of the Gated DeltaNet token mixer.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only
the tests, the smoke check and the benchmark's CPU-baseline leg do.  It shares
no code with the CUDA path.

* ``forward`` / ``decode_step``: the plain token-by-token recurrence in fp64
  (C, threaded over (batch, V head)) -- the definition the GPU results are
  checked against.
* ``chunk_forward``: an fp64 numpy restatement of the chunkwise WY form, used
  by the tests as an independent reformulation that must agree with it.
* ``backward``: fp64 gradients of every input (the adjoint of the token
  recurrence), for the backward pass.
* ``chunk_backward``: the same gradients through the chunkwise WY form (the
  blocked algebra of a chunked backward kernel), required to agree with it.
"""
from .oracle import decode_step, default_threads, forward  # noqa: F401
from .chunk_form import chunk_forward  # noqa: F401
from .backward import backward  # noqa: F401
from .chunk_backward import chunk_backward  # noqa: F401
