"""Exact IO-aware attention on B200 (sm_100a)."""
