"""CPU oracle for hash-scored top-k sparse decode attention.

TEST INFRASTRUCTURE. This package is the slow, plain, obviously-correct
reference that the CUDA library is checked against. Only the test suite,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path (the C-ABI library and
its Python binding) never imports, calls or links anything here, and nothing
here imports the product path.

Everything is computed in float64 with numpy, one (batch, kv-head) pair at a
time. Where numpy supplies a primitive (a matrix product, a stable sort) it
is used as one step; there is no blocking, fusion or reordering beyond what
the pages' definitions state.

Sources, cited by page title and section:

* SOCKET technical summary -- "SOCKET - SOft Collision Kernel EsTimator for
  sparse attention" (gist.science/ja/paper/2602.06283), section
  "中核メカニズム：ソフト LSH" (core mechanism: soft LSH), steps 1-4, and
  section "理論的基盤" (theoretical foundation) for the tau -> 0 limit.
* HATA digest -- "HATA: Hash-Aware Top-k Attention" (aibr.jp/archives/117328),
  section 3 "中核となる技術的要素" (binary hash codes compared to rank keys).
* SOCKET technical summary, "主要な貢献" item 4 and "理論的基盤": the
  soft-count attention estimator (``estimator_ref``).
* Tactic digest -- "Tactic: Adaptive Sparse Attention with Clustering and
  Distribution Fitting for Long-Context LLMs" (aibr.jp/archives/79195),
  section 3 "中核となる技術的要素" (the cumulative score target): the
  adaptive k, and per-query-head index sets (``selection_ref``).
* HATA digest, sections 3 and 4 (the offloaded KV cache), and the HGA page,
  section 3 (hot and routed pages): the paged / host-resident K/V pool
  (``paged_ref``).

Pins. Every public function below is named in a ``-m "not gpu"`` test that
a plausible slip in it would fail; the expected values there are closed
forms, hand-built fixtures, brute force or scipy routines, never this
package's own output:

* hash_key_ids, value_norms_f16, bucket_probabilities, group_bucket_table,
  soft_collision_scores, select_topk, socket_decode_pair:
  ``tests/test_oracle_socket.py`` (basis-vector fixtures, negation and scale
  invariance, fsum brute force, the bit-factorisation identity, the tau
  limits, brute-force top-k with ties, k = N against scipy's softmax);
* exact_attention, attend_subset, dense_decode, binary_codes,
  hamming_match_scores: ``tests/test_oracle_attention_hata.py``;
* hata_decode_pair, socket_decode, hata_decode (the compositions and the
  query-head -> KV-head mapping): ``tests/test_oracle_compositions.py``;
* soft_counts, soft_count_attention: ``tests/test_oracle_estimator.py``
  (a one-hyperplane case worked with math.exp, the tau -> infinity limit, a
  pure-Python loop over tables and buckets);
* per_head_scores, socket_decode_pair_per_head, adaptive_k, select_adaptive,
  socket_decode_pair_adaptive: ``tests/test_oracle_selection.py`` (uniform
  and geometric closed forms, hand-built ties and clamps, a pure-Python
  greedy loop, the one-head and equal-heads reductions, scipy's softmax);
* paged_rows, attend_subset_paged, socket_decode_pair_paged:
  ``tests/test_oracle_paged.py`` (a hand-built pool, the identity and
  permuted page tables against the contiguous functions, page size 1 and one
  page per pair, scipy's softmax).
"""

from .socket_ref import (
    hash_key_ids,
    value_norms_f16,
    bucket_probabilities,
    group_bucket_table,
    soft_collision_scores,
    select_topk,
    socket_decode_pair,
    socket_decode,
)
from .attention_ref import exact_attention, attend_subset, dense_decode
from .hata_ref import binary_codes, hamming_match_scores, hata_decode_pair, hata_decode
from .estimator_ref import soft_counts, soft_count_attention
from .selection_ref import (
    per_head_scores,
    socket_decode_pair_per_head,
    adaptive_k,
    select_adaptive,
    socket_decode_pair_adaptive,
)
from .paged_ref import paged_rows, attend_subset_paged, socket_decode_pair_paged

__all__ = [
    "hash_key_ids",
    "value_norms_f16",
    "bucket_probabilities",
    "group_bucket_table",
    "soft_collision_scores",
    "select_topk",
    "socket_decode_pair",
    "socket_decode",
    "exact_attention",
    "attend_subset",
    "dense_decode",
    "binary_codes",
    "hamming_match_scores",
    "hata_decode_pair",
    "hata_decode",
    "soft_counts",
    "soft_count_attention",
    "per_head_scores",
    "socket_decode_pair_per_head",
    "adaptive_k",
    "select_adaptive",
    "socket_decode_pair_adaptive",
    "paged_rows",
    "attend_subset_paged",
    "socket_decode_pair_paged",
]
