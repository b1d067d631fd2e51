"""fp64 CPU oracle for FlashBlock denoise-step attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may use it.  It shares no code with the CUDA library; the only
module both consume is the seeded input generator
(``cached_split_attention_b200.workloads``), which draws inputs and holds none of
the method's arithmetic.

Contents
  attention.py  the plain definition of softmax attention over a key set, with its
                log-normaliser (FlashBlock, "Mecanismo Central"), and the log-space
                merge of two partials (FlashBlock, the A_full equation of
                "Mecanismo Central").
  policy.py     the reuse gates (FlashBlock, "Estrategias de Reutilizacion
                Adaptativa": threshold tau on the updated-token count and the
                per-head similarity gate gamma; SureLock, "Mecanismo de
                Funcionamiento": locked rows compute no query) and the step-by-step
                policy that keeps the (A_out, L_out) cache.
  brute.py      pure-Python (math.fsum) restatement of the definition, used to pin
                attention.py on tiny inputs.
  transition.py the block transition: a finished block's K/V join each sequence's
                prefix (FlashBlock, "Mecanismo Central": finished tokens become
                out-of-block context) and the next block starts from an empty cache.
  sparse.py     the sparse-residual variant (FlashBlock, "Estrategias de Reutilizacion
                Adaptativa", third bullet): keys a sparse pattern leaves out form the
                cached out-of-block set; the selected ones join the block's keys.

Pins: every function here is checked in ``tests/test_oracle_*.py`` against brute
force, closed forms, the merge identities and hand-derived fixtures under
``tests/golden/``.  The approximate outputs of *reuse* steps have no external truth
on the pages (they print no error figures): parity unpinned for the size of the
reuse approximation error, which the oracle reports for information only.
"""
from .attention import attend, attend_problem, bf16_to_f64, merge  # noqa: F401
from .policy import OracleCache, decide, head_cosine, run_policy  # noqa: F401
from . import sparse, transition  # noqa: F401
