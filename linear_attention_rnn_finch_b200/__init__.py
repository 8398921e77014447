"""B200 (sm_100a) WKV6 recurrence: chunked prefill and decode step behind a C ABI."""
