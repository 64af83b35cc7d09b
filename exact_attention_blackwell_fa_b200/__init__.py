"""Exact scaled-dot-product attention (forward and backward) for B200 / sm_100a."""
