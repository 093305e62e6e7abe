"""Seeded synthetic inputs (shared by tests, oracle callers and the benchmark)."""
