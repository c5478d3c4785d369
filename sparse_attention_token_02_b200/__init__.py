"""DeepSeek Sparse Attention Lightning Indexer on B200 (sm_100a).

The CUDA library (libdsa_indexer.so, built by ``python -m sparse_attention_token_02_b200.build``)
does all the work; ``api`` marshals torch tensors into its C ABI and ``workloads`` draws
the seeded synthetic inputs.
"""

__all__ = ["api", "workloads"]
