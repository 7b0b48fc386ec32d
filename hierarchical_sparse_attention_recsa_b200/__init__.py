"""RecSA hot path on B200: a C-ABI library (``librecsa.so``, declared in
include/recsa.h) and its Python binding (``recsa``).

A decode loop, with the caller owning every device buffer::

    import torch
    from hierarchical_sparse_attention_recsa_b200 import recsa as R

    g = R.Geometry(head_dim=128, n_q_heads=32, n_kv_heads=8, leaf_block=64,
                   branching=16, k=8, window=512, batch=4, capacity=cap)
    tree = torch.zeros(R.recsa_tree_bytes(g), dtype=torch.uint8, device="cuda")
    R.recsa_build(g, K, V, lens_host, r, 0, tree)          # pool the whole cache
    for step in range(n):                                   # one launch per step
        R.recsa_decode_step(g, Q[step], K, V, k_new[step], v_new[step], lens,
                            r, 0, tree, 1, O)
    R.recsa_prefill(g, Qp, K, V, tree, q_start, n_q, Op)    # causal queries

K, V are [batch][n_kv_heads][capacity][head_dim] (bf16 or fp32), Q and O
[batch][n_q][n_q_heads][head_dim], ``lens`` an int64 device tensor of the
sequence lengths, ``r`` the pooler's reference vector(s).  The geometry's
``mode`` selects RecSA (default), ZHA top-p routing (``mode=R.MODE_ZHA,
top_p=...``, optionally ``n_ref`` reference queries and ``key_format`` FP8 or
NVFP4 router keys) or one selection per KV group (``mode=R.MODE_GROUP``).

``synth`` generates the seeded synthetic workloads, ``counts`` the work
accounting used by the benchmark, ``build_lib`` compiles the library in-tree.
"""
