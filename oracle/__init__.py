"""CPU oracle for SageSLA attention -- test infrastructure only (see oracle.c)."""
