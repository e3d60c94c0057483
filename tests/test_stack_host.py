"""Host logic of the layer stack, without a GPU: which layers run a chunk
after cached tokens on their own window workspace (a KV-shared local layer
and its source), and the workspace sizes the stack asks the library for."""
from hybrid_local_global_b200 import native
from hybrid_local_global_b200.stack import AttentionStack
from hybrid_local_global_b200.workloads import L31B_GLOBAL, L31B_LOCAL, WORKLOADS, Workload


def test_window_sources_of_the_12_layer_shared_stack():
    """12 layers at 5:1 with the last 2 shared: layer 10 (local) shares
    layer 9, layer 11 (global) shares layer 5. Only the local pair takes a
    window workspace, and only after cached tokens."""
    w = Workload("shared12", "decode", batch=1, n_q_heads=32, n_layers=12, ratio=5, local=L31B_LOCAL,
                 global_=L31B_GLOBAL, len_lo=1, len_hi=256, n_shared=2)
    st = AttentionStack(w, "cpu")  # small host caches: a share binding needs its source's
    assert st.descs[10].shared_from == 9 and st.descs[11].shared_from == 5
    assert st._window_source(10, True) == 9
    assert st._window_source(9, True) == 9          # the source leaves its window
    assert st._window_source(11, True) is None      # a global layer re-reads nothing it lost
    assert st._window_source(5, True) is None
    assert st._window_source(8, True) is None       # a local layer nobody shares
    assert st._window_source(10, False) is None     # no cached tokens: the ring holds everything


def test_window_sources_without_sharing():
    st = AttentionStack(WORKLOADS["31b_verify_b64_k4"], "cpu", alloc_caches=False)
    assert all(st._window_source(l, True) is None for l in range(st.n_layers))


def test_multi_token_workspace_covers_every_layer():
    st = AttentionStack(WORKLOADS["31b_verify_b64_k4"], "cpu", alloc_caches=False)
    n = st.decode_multi_workspace_bytes(4, 131072)
    for l in range(st.n_layers):
        t = st.layer_type(l)
        cap = t.window if t.window else st.global_capacity
        assert n >= native.gemma_attn_decode_multi_workspace_size(64, 4, 32, t.n_kv_heads, t.head_dim, t.window,
                                                                  131072, cap, 0)
