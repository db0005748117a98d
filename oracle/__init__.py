"""fp64 CPU oracle for the lightning-indexer selection path -- TEST INFRASTRUCTURE.

This package is a plain, slow, obviously-correct restatement of what the
selection path computes.  It exists only to check the CUDA library: the tests,
the package's ``smoke()`` check and the benchmark's CPU-baseline leg are the
only code allowed to import it.  It shares no code, headers or tables with the
CUDA library and never imports it.

Sources (page title, section):

* Indexer score: "03 long context" lecture, section "The Architectural Answer:
  Read Less of the Past" (DSA stage 1, the lightning indexer: one shared
  128-d key per position scored by a weighted-ReLU dot product over the query
  heads); "Latent Sparse Attention", section "Where the time goes" (a
  GLM-shaped indexer of 32 heads x 128 dims that applies ReLU and the head
  weights and keeps its top 512).  The pages never print the formula; the
  reading used is score(t, s) = sum_h w[t, h] * max(0, q[t, h] . k[s]).
* Stride-4 compression and causal eligibility: LeanSparse podcast transcript,
  02:36-02:56; "03 long context", section "DeepSeek-V4: Compress the History,
  Then Sparsify It".
* Top-k with ties to the lower position: "Latent Sparse Attention", section
  "What the kernels do about the top-p" (packed keys with the score above the
  inverted id).
* Two-stage decode search: LeanSparse podcast transcript, 07:12-08:00.
* Sparse main attention over the selected rows (absorbed MLA: the 576-element
  latent row is the key of every head, its first 512 elements the value):
  "03 long context", section "The Architectural Answer: Read Less of the
  Past" (stage 2) and "Derivation 6" (576-element bf16 latent rows).
* Bucket search: "Latent Sparse Attention", sections "How LSA finds the keys"
  and "The method, term by term" (steps 5 and 6).

Modules: ``formats`` (byte formats), ``indexer`` (scores, eligibility),
``select`` (top-k and the three search pipelines), ``attention`` (sparse
main attention and the online-softmax merge), ``brute`` (pure-Python
loops for tiny inputs), ``sizes`` (the pages' size arithmetic).
"""

from .formats import bf16_to_f64, e4m3_to_f64  # noqa: F401
from .indexer import indexer_scores, eligible_count  # noqa: F401
from .select import (  # noqa: F401
    topk_rows,
    select_topk,
    decode_select,
    prefill_select,
    two_stage_select,
    bucket_select,
    recall_at_k,
)
