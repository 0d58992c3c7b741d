"""Paged KV-cache decode attention for one B200 (sm_100a)."""
