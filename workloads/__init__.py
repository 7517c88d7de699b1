"""Seeded synthetic inputs shared by the tests and the benchmark (no method arithmetic)."""
