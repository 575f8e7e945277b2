"""Float64 CPU oracle for causal factorized sparse self-attention.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plain, obviously
correct statement of what the GPU library computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product path
(``factorized_block_sparse_b200``) never imports, links or executes
anything in here, and nothing in here imports the product path: the two
share no code, only the seeded input generator
(``factorized_block_sparse_b200.synth``), which holds none of the method's
arithmetic.

Sources (web pages on the Sparse Transformer; cited by title and section):

* "OpenAI Sparse Transformer" (agentlenshq blog), sections "Reducing Memory
  Constraints with Deep Attention", "Sparse Attention and Algorithmic
  Complexity", "Factorized Attention Patterns", "Implementation and
  Limitations".
* "[논문 리뷰] Generating Long Sequences with Sparse Transformers" (nubint
  review), sections "ABSTRACT" and "제안 방법".
* "Генеративное моделирование с разреженными трансформерами (sparse
  transformers)" (pcnews translation of the OpenAI post), sections
  "Глубокое внимание", "Разреженное внимание", "Релиз кода".
* "Insights: 희소 어텐션 (Sparse Attention)" (molayo), the paragraphs on the
  ``SparseAttention`` class and ``attention_impl`` /
  ``blocksparse_attention_impl`` with modes "all", "local", "strided".

Modules:

* ``patterns``  - element-level masks of the four modes and their
  component heads.
* ``views``     - the split of each pattern into views that are dense in
  some relabelled order, and the block look-up tables (block-OR of the
  element masks).
* ``attention`` - masked softmax attention and its analytic gradient in
  float64, whole tensors or sampled rows / key columns.

Every function is pinned by ``-m "not gpu"`` tests against something other
than itself (library attention with autograd, finite differences,
closed-form counts, two-step reachability, special cases, brute force on
tiny inputs).  No function here is "parity unpinned".
"""

from . import patterns, views, attention  # noqa: F401

MODES = ("all", "local", "strided", "fixed")
