"""M-FALCON masked prefill attention, KV pool write and cross-stage rank decode on B200 (sm_100a)."""
