"""Paged and host-offloaded KV gather -- float64 CPU oracle.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Sources: the HATA digest ("HATA: Hash-Aware Top-k Attention",
aibr.jp/archives/117328), sections 3 and 4: its offloading variant keeps the
KV cache in host memory behind PCIe and brings in only the keys and values it
needs; and the HGA page (Hierarchical Global Attention explainer,
gist.science/ja/paper/2606.30709), section 3: only the recent ("hot") pages
and the routed older pages of the cache are held close to the compute.
Neither prints a layout. The reading used here, the plainest one: the K and
V rows of every (batch, KV-head) pair live in a pool of fixed-size pages,

    K_pool, V_pool: [num_pages][page_size][d],

and a page table [B][Hkv][max_pages] maps the pair's logical page p (keys
p * page_size .. p * page_size + page_size - 1) to a physical page. Key n of
a pair is row n % page_size of page page_table[pair][n // page_size]. The
pool may live in device memory or in pinned host memory; the result does not
depend on where. Attention over a selected subset is then the exact subset
attention of ``attention_ref.attend_subset`` over the gathered rows.
"""

from __future__ import annotations

import numpy as np

from .attention_ref import attend_subset
from .socket_ref import group_bucket_table, select_topk, soft_collision_scores


def paged_rows(pool, page_table_pair, idx, page_size: int) -> np.ndarray:
    """Rows of keys idx of one pair: pool[page_table_pair[n // page_size], n % page_size]."""
    idx = np.asarray(idx, dtype=np.int64)
    pages = np.asarray(page_table_pair, dtype=np.int64)[idx // page_size]
    return np.asarray(pool, dtype=np.float64)[pages, idx % page_size]


def attend_subset_paged(Qg, K_pool, V_pool, page_table_pair, idx, page_size: int, scale: float) -> np.ndarray:
    """Exact attention of the G query heads over keys idx, read from the pools."""
    idx = np.asarray(idx, dtype=np.int64)
    K = paged_rows(K_pool, page_table_pair, idx, page_size)
    V = paged_rows(V_pool, page_table_pair, idx, page_size)
    return attend_subset(Qg, K, V, np.arange(len(idx)), scale)


def socket_decode_pair_paged(Qg, K_pool, V_pool, page_table_pair, page_size, R, ids, norms, L, P, tau, k, scale):
    """The decode step of one pair with a paged K/V cache: steps 2-4 select
    from the (contiguous) hashed-key cache, the attention reads the pages.
    Returns (O [G, d], idx [k], scores [N])."""
    scores = soft_collision_scores(group_bucket_table(Qg, R, L, P, tau), ids, norms)
    idx = select_topk(scores, k)
    return attend_subset_paged(Qg, K_pool, V_pool, page_table_pair, idx, page_size, scale), idx, scores
