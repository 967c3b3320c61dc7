"""EntmaxKV support-aware paged α-entmax decode for B200 (sm_100a).

The compute path is the C-ABI library ``libekv.so`` (hand-written CUDA);
``binding`` marshals PyTorch tensors into its calls.
"""
