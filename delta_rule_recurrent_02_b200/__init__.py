"""B200 (sm_100a) causal delta-rule layer: chunked prefill and decode step."""
