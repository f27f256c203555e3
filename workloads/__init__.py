"""Seeded synthetic workload generators shared by the tests, the oracle checks and the bench."""
