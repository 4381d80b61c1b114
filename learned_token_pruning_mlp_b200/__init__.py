"""B200-native (sm_100a) library for the TokenGate pruned-prefill hot path."""
