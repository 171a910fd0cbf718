"""Gated delta rule forward pass and decode step for B200 (sm_100a)."""
