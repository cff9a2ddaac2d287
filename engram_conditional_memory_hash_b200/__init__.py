"""Engram conditional-memory hot path for B200 (sm_100a)."""
