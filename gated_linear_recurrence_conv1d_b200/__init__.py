"""RG-LRU recurrent block (causal conv1d -> RG-LRU -> GeLU merge) on B200 (sm_100a)."""
